"""The perturbed layer outputs (dust_noisy_linear_output) against the oracle's noise and an
exact fp64 product of the stored inputs.  fp32 output: fp32 accumulation of exact bf16
products plus sigma times an fp32 normal within 1e-5 of exact, so |err| <= 1e-5 (1 + |y|);
bf16 output: within one bf16 rounding (2^-8 relative) of that."""
import numpy as np
import pytest

import oracle
import workloads
from tests import _dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as zz
    zz.lib()
    return zz


@pytest.mark.parametrize("N,d_in,d_out,K", [(200, 64, 48, 3), (300, 256, 528, 2), (1, 16, 16, 1)])
def test_noisy_output_matches_oracle(z, N, d_in, d_out, K):
    import torch
    L = workloads.custom_layer(N + d_out, N, d_in, d_out, "bf16", 0.05)
    x, W, _ = _dev.layer_to_device(L)
    key = z.NoiseKey(0x5EED00B1, layer_id=5, draw_offset=7, token_offset=1000, channel_offset=0)
    sigma = 1e-2
    y = z.dust_noisy_linear_output(x, W, K, sigma, key)
    yb = z.dust_noisy_linear_output(x, W, K, sigma, key, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    a = oracle.noise(key.seed, 5, N, d_out, K, draw_offset=7, token_offset=1000)
    ref = (L.x_f64 @ L.W_f64.T)[None] + sigma * a
    got = _dev.host(y).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * (1 + np.abs(ref)))
    gb = _dev.host(yb.float()).astype(np.float64)
    assert np.all(np.abs(gb - ref) <= 2.0**-8 * np.abs(ref) + 1e-5 * (1 + np.abs(ref)))


def test_noisy_output_gives_the_forward_loss_change(z):
    """The quadratic readout of the materialised outputs reproduces the fused forward's loss
    change (the same noise for the same key)."""
    import torch
    N, d_in, d_out, K, sigma = 256, 128, 256, 4, 1e-3
    L = workloads.custom_layer(91, N, d_in, d_out, "bf16", 0.02)
    x, W, u = _dev.layer_to_device(L)
    key = z.NoiseKey(0x5EED00B2, layer_id=2)
    y = z.dust_noisy_linear_output(x, W, K, sigma, key)
    dl = z.dust_noisy_linear_fwd(x, W, u, K, sigma, key)
    torch.cuda.synchronize()
    yh = _dev.host(y).astype(np.float64)
    clean = L.x_f64 @ L.W_f64.T - L.u_f64
    loss = 0.5 * ((yh - L.u_f64[None]) ** 2).sum(-1) - 0.5 * (clean ** 2).sum(-1)[None]
    _, ref_clean = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, K, sigma, key.seed, 2)
    lo, _ = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, K, sigma, key.seed, 2)
    # both against the oracle: the outputs' loss change (loose: a difference of large fp32
    # numbers) and the fused forward's (tight)
    assert np.abs(loss - (lo - ref_clean)).max() <= 1e-3 * np.abs(lo - ref_clean).max() + 1e-3
    _dev.assert_fp32_close(_dev.host(dl), lo - ref_clean, "fused forward")
