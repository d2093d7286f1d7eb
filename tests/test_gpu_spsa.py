"""SPSA / MeZO weight-space probe (the contrast estimator) on the GPU against the oracle.
The projected gradient p_j = (L_+ - L_-) / (2 eps) is a random projection of the gradient G
and can be near zero, so it is compared on the scale of |G|_F: |p_gpu - p_ref| <= 2e-3 |G|_F
(the GPU's bf16 directions equal the oracle's except where its fp32 normal, within 1e-5 of the
exact one, lands on the other side of a bf16 rounding boundary; fp32 sums).  The losses
L_+- are sums of positive terms: relative 1e-4.  The estimate: relative Frobenius 2e-3."""
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


def _gradient(L):
    E = L.x_f64 @ L.W_f64.T - L.u_f64
    return E.T @ L.x_f64


@pytest.mark.parametrize("N,d_in,d_out,P", [(200, 64, 48, 5), (300, 256, 512, 3),
                                            (129, 16, 272, 2)])
def test_spsa_probe_matches_oracle(z, N, d_in, d_out, P):
    import torch
    L = workloads.custom_layer(N + d_out, N, d_in, d_out, "bf16", 0.05)
    x, W, u = _dev.layer_to_device(L)
    key = z.NoiseKey(0x5EED0008, layer_id=4, draw_offset=11)
    p, Lp, Lm = z.dust_spsa_probe(x, W, u, P, 1e-3, key, losses=True)
    torch.cuda.synchronize()
    pr, Lpr, Lmr = oracle.spsa_probe(L.x_f64, L.W_f64, L.u_f64, P, 1e-3, key.seed, 4, 11)
    scale = np.linalg.norm(_gradient(L))
    assert np.abs(_dev.host(p) - pr).max() <= 2e-3 * scale, (_dev.host(p), pr, scale)
    np.testing.assert_allclose(_dev.host(Lp), Lpr, rtol=1e-4)
    np.testing.assert_allclose(_dev.host(Lm), Lmr, rtol=1e-4)


def test_spsa_estimate_matches_oracle_and_chunks_add_up(z):
    import torch
    d_out, d_in, P = 96, 128, 7
    key = z.NoiseKey(0x5EED0009, layer_id=6, draw_offset=2)
    p = np.random.default_rng(3).standard_normal(P).astype(np.float32)
    pt = torch.from_numpy(p).cuda()
    G = z.dust_spsa_estimate(pt, P, d_out, d_in, key)
    Gc = z.dust_spsa_estimate(pt[:3], P, d_out, d_in, key)
    z.dust_spsa_estimate(pt[3:], P, d_out, d_in, key._replace(draw_offset=5), G=Gc,
                         accumulate=True)
    torch.cuda.synchronize()
    ref = oracle.spsa_estimate(p.astype(np.float64), P, d_out, d_in, key.seed, 6, 2)
    assert _dev.rel_fro(_dev.host(G), ref) <= _dev.GW_FRO
    np.testing.assert_allclose(_dev.host(Gc), _dev.host(G), rtol=1e-5, atol=1e-6)


def test_spsa_token_shards_sum_to_the_whole_batch(z):
    """With tokens split over devices each shard's p is a partial sum: P scalars to exchange."""
    import torch
    N, d_in, d_out, P = 512, 128, 256, 4
    L = workloads.custom_layer(77, N, d_in, d_out, "bf16", 0.05)
    x, W, u = _dev.layer_to_device(L)
    key = z.NoiseKey(0x5EED000B, layer_id=1)
    whole = _dev.host(z.dust_spsa_probe(x, W, u, P, 1e-3, key))
    a = _dev.host(z.dust_spsa_probe(x[:200].contiguous(), W, u[:200].contiguous(), P, 1e-3, key))
    b = _dev.host(z.dust_spsa_probe(x[200:].contiguous(), W, u[200:].contiguous(), P, 1e-3, key))
    scale = np.linalg.norm(_gradient(L))
    assert np.abs(a + b - whole).max() <= 1e-5 * scale


def test_spsa_rejects_bad_arguments(z):
    import torch
    x = torch.zeros((8, 16), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(z.DustError):
        z.dust_spsa_probe(x, W, x, 2, 1e-3, z.NoiseKey(1, layer_id=0x80000000))
    with pytest.raises(z.DustError):
        z.dust_spsa_probe(x, W, x, 2, 0.0, z.NoiseKey(1))
    with pytest.raises(z.DustError):
        z.dust_spsa_probe(x.float(), W.float(), x.float(), 2, 1e-3, z.NoiseKey(1))
