"""Optimizer steps on the weight estimate (SGD with momentum, Adam): the standalone kernel
against the oracle, and the step fused into the contraction's last pass against the
unfused sequence.  Tolerances: the step is elementwise fp32 arithmetic on inputs the oracle
reads exactly.  W and v (sums of same-signed terms) are within a few fp32 ulps of the fp64
result (rtol 2e-6).  The momentum m is a short sum of gradients that can cancel, so its
error is bounded by the terms' magnitudes, not by m: |err| <= 8 * 2^-24 * M, where M is the
same recurrence run on |G| (each of the <= 3 steps rounds a product and a sum)."""
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


def _f32(x: float) -> float:
    return float(np.float32(x))


def _t(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


@pytest.mark.parametrize("kind", ["sgd", "adam"])
@pytest.mark.parametrize("n", [4096, 10003])
def test_optimizer_step_matches_oracle(z, kind, n):
    import torch
    rng = np.random.default_rng(5)
    W0 = rng.standard_normal(n).astype(np.float32)
    W, m, v = _t(W0), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    Wb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    Wr, mr, vr = W0.astype(np.float64), np.zeros(n), np.zeros(n)
    M = np.zeros(n)   # the momentum recurrence on |G|: the size of the terms m sums
    for t in range(1, 4):
        G = (rng.standard_normal(n) * 0.1).astype(np.float32)
        M = (0.9 * M + np.abs(G)) if kind == "sgd" else (0.9 * M + 0.1 * np.abs(G))
        # the call's hyper-parameters are fp32 (dust_opt_params); the oracle reads those values
        if kind == "sgd":
            z.dust_optimizer_step(z.sgd_momentum(0.05, 0.9, 0.01), _t(G), W, m, W_bf16=Wb)
            Wr, mr = oracle.sgd_momentum(Wr, mr, G, _f32(0.05), _f32(0.9), _f32(0.01))
        else:
            z.dust_optimizer_step(z.adam(1e-3, t, weight_decay=0.01), _t(G), W, m, v, W_bf16=Wb)
            Wr, mr, vr = oracle.adam(Wr, mr, vr, G, _f32(1e-3), _f32(0.9), _f32(0.999),
                                     _f32(1e-8), t, _f32(0.01))
    torch.cuda.synchronize()
    np.testing.assert_allclose(_dev.host(W), Wr, rtol=2e-6, atol=1e-7)
    assert np.all(np.abs(_dev.host(m) - mr) <= 8 * 2.0**-24 * M)
    if kind == "adam":
        np.testing.assert_allclose(_dev.host(v), vr, rtol=2e-6, atol=1e-12)
    assert torch.equal(Wb, W.to(torch.bfloat16))


@pytest.mark.parametrize("kind", ["sgd", "adam"])
@pytest.mark.parametrize("N,d_in,d_out", [(4100, 256, 256), (1024, 2048, 2048)])
def test_fused_step_equals_weight_grad_then_step(z, kind, N, d_in, d_out):
    """Both the split-K path (small output) and the single-pass path (large output)."""
    import torch
    K = 8
    L = workloads.custom_layer(40 + d_out, N, d_in, d_out, "bf16", 0.02)
    x = _dev.to_device(L.x_store, "bf16")
    r = _t(workloads.gaussian_losses(41, K, N, scale=0.05))
    key = z.NoiseKey(0x5EED0002, layer_id=3)
    rng = np.random.default_rng(6)
    W0 = _t(rng.standard_normal((d_out, d_in)) * 0.02)
    m0 = _t(rng.standard_normal((d_out, d_in)) * 1e-3)
    v0 = _t(np.abs(rng.standard_normal((d_out, d_in))) * 1e-6)
    opt = z.sgd_momentum(0.01, 0.9) if kind == "sgd" else z.adam(1e-3, 3)
    # unfused
    Wa, ma, va = W0.clone(), m0.clone(), v0.clone()
    Ga, _ = z.dust_weight_grad(r, x, d_out, K, 1e-3, key)
    z.dust_optimizer_step(opt, Ga, Wa, ma, va)
    # fused, with and without storing G_W
    Wf, mf, vf = W0.clone(), m0.clone(), v0.clone()
    Gf = torch.empty_like(Ga)
    Wbf = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    z.dust_weight_grad_step(r, x, d_out, K, 1e-3, key, opt, Wf, mf, vf, W_bf16=Wbf, G_W=Gf)
    Wn, mn, vn = W0.clone(), m0.clone(), v0.clone()
    z.dust_weight_grad_step(r, x, d_out, K, 1e-3, key, opt, Wn, mn, vn)
    torch.cuda.synchronize()
    assert torch.equal(Gf, Ga)
    for a, b in ((Wf, Wa), (mf, ma), (vf, va), (Wn, Wa), (mn, ma)):
        np.testing.assert_allclose(_dev.host(a), _dev.host(b), rtol=2e-6, atol=1e-9)
    assert torch.equal(Wbf, Wf.to(torch.bfloat16))


def test_fused_sgd_step_matches_oracle_chain(z):
    """The whole update W1 - W0 = -lr (mu m0 + G_W) against the oracle's G_W (2e-3)."""
    import torch
    N, d_in, d_out, K, sigma = 1000, 128, 256, 8, 1e-3
    L = workloads.custom_layer(42, N, d_in, d_out, "bf16", 0.02)
    r = workloads.gaussian_losses(43, K, N, scale=0.05)
    key = z.NoiseKey(0x5EED0002)
    W0 = np.zeros((d_out, d_in), np.float32)
    W, m = _t(W0), torch.zeros((d_out, d_in), device="cuda")
    z.dust_weight_grad_step(_t(r), _dev.to_device(L.x_store, "bf16"), d_out, K, sigma, key,
                            z.sgd_momentum(0.1, 0.9), W, m)
    torch.cuda.synchronize()
    g = oracle.output_error(r, K, sigma, key.seed, d_out)
    Wr, _ = oracle.sgd_momentum(W0, np.zeros_like(W0), oracle.weight_grad(g, L.x_f64), 0.1, 0.9)
    assert _dev.rel_fro(_dev.host(W), Wr) <= _dev.GW_FRO


def test_optimizer_rejects_bad_parameters(z):
    import ctypes
    bad = [z.sgd_momentum(0.1, 1.0), z.adam(1e-3, 0), z.adam(-1.0, 1),
           z.dust_opt_params(7, 1, 0.1, 0, 0, 0, 0, 0)]
    buf = _t(np.zeros(16))
    for p in bad:
        assert z.lib().dust_optimizer_step(ctypes.byref(p), buf.data_ptr(), buf.data_ptr(), None,
                                           buf.data_ptr(), buf.data_ptr(), 16, None) == \
            z.DUST_ERR_INVALID_ARG
