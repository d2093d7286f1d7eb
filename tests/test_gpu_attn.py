"""Attention-internal reward (Dust page, "간섭(interference) 줄이기"): the CUDA reward and the
credit equation without centring against the oracle, and the whole estimate of a value
projection from the reward.  Tolerances: the reward is an fp32 dot product of exactly read
inputs (element error <= 1e-3 x RMS, relative Frobenius <= 1e-4); the scan is bit-exact on
dyadic rewards and within the general-gamma bound otherwise; g and G_W 2e-3."""
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


def _dO(rng, K, N, d, ld, dtype):
    """delta_o [K, N, ld] (columns d..ld-1 are padding, filled with NaN) as stored and as f64."""
    import torch
    a = (rng.standard_normal((K, N, d)) * 1e-3).astype(np.float32)
    if dtype == "bf16":
        bits = workloads.to_bf16_bits(a)
        a64 = workloads.bf16_bits_to_f64(bits)
        full = np.full((K, N, ld), 0x7FC0, dtype=np.uint16)
        full[:, :, :d] = bits
        t = torch.from_numpy(full.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        a64 = a.astype(np.float64)
        full = np.full((K, N, ld), np.nan, dtype=np.float32)
        full[:, :, :d] = a
        t = torch.from_numpy(full).cuda()
    return t[:, :, :d], a64


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,K,pad", [(1, 8, 1, 0), (333, 200, 3, 8), (64, 768, 17, 0),
                                       (1000, 64, 16, 16)])
def test_attn_reward_matches_oracle(z, dtype, N, d, K, pad):
    import torch
    rng = np.random.default_rng(N + d + K)
    G = rng.standard_normal((N, d)).astype(np.float32)
    dO, dO64 = _dO(rng, K, N, d, d + pad, dtype)
    c = z.dust_attn_reward(torch.from_numpy(G).cuda(), dO)
    torch.cuda.synchronize()
    _dev.assert_fp32_close(_dev.host(c), oracle.attn_reward(G.astype(np.float64), dO64),
                           "reward")


@pytest.mark.parametrize("gamma", [0.0, 1.0])
@pytest.mark.parametrize("K", [1, 5, 130])
def test_discounted_credit_bit_exact_on_dyadic_rewards(z, gamma, K):
    import torch
    N = 3000
    c = workloads.dyadic_losses(7 + K, K, N)
    cu = workloads.random_segments(8, N, 1, 600)
    r = z.dust_discounted_credit(torch.from_numpy(c).cuda(), _dev.cu_to_device(cu), gamma)
    torch.cuda.synchronize()
    ref = oracle.discounted_credit(c, cu, gamma)
    assert np.array_equal(_dev.host(r).astype(np.float64), ref)


def test_discounted_credit_general_gamma(z):
    import torch
    K, N, gamma = 8, 5000, 0.99
    c = workloads.gaussian_losses(9, K, N)
    cu = workloads.random_segments(10, N, 256, 2048)
    r = _dev.host(z.dust_discounted_credit(torch.from_numpy(c).cuda(), _dev.cu_to_device(cu),
                                           gamma))
    ref = oracle.discounted_credit(c, cu, gamma)
    L = np.diff(cu).max()
    bound = 2e-6 * (min(L, 1.0 / (1.0 - gamma)) + 1) * np.abs(ref).max() + 1e-6
    assert np.abs(r - ref).max() <= bound


def test_value_projection_estimate_from_the_reward(z):
    """A value projection v = W_V x perturbed per token; a causal mixing P turns it into the
    attention output, so delta_o = sigma P a; the reward, the credit (gamma = 1 within each
    sequence) and the output-error / weight-estimate equations give g and G_W of W_V."""
    import torch
    N, d_model, d, K, sigma = 256, 64, 128, 8, 1e-3
    key = z.NoiseKey(0x5EED00A7, layer_id=3)
    rng = np.random.default_rng(12)
    seq = np.array([0, 100, 256], dtype=np.int32)
    P = np.zeros((N, N))
    for a, b in zip(seq[:-1], seq[1:]):
        blk = np.tril(rng.random((b - a, b - a)) + 0.1)
        P[a:b, a:b] = blk / blk.sum(1, keepdims=True)
    noise = oracle.noise(key.seed, 3, N, d, K)                  # the value projection's noise
    dO64 = sigma * np.einsum("st,itk->isk", P, noise)
    dO = torch.from_numpy(dO64.astype(np.float32)).cuda()
    G = rng.standard_normal((N, d)).astype(np.float32)          # error at the attention output
    X = workloads.custom_layer(13, N, d_model, d, "bf16")      # the projection's input x
    c = z.dust_attn_reward(torch.from_numpy(G).cuda(), dO)
    r = z.dust_discounted_credit(c, _dev.cu_to_device(seq), 1.0)
    GW, g = z.dust_weight_grad(r, _dev.to_device(X.x_store, "bf16"), d, K, sigma, key,
                               g_out=True)
    torch.cuda.synchronize()
    c_ref = oracle.attn_reward(G.astype(np.float64), dO.cpu().numpy().astype(np.float64))
    r_ref = oracle.discounted_credit(c_ref, seq, 1.0)
    g_ref = oracle.output_error(r_ref, K, sigma, key.seed, d, 3)
    assert _dev.rel_fro(_dev.host(g), g_ref) <= _dev.GW_FRO
    assert _dev.rel_fro(_dev.host(GW), oracle.weight_grad(g_ref, X.x_f64)) <= _dev.GW_FRO


def test_attn_reward_rejects_bad_layouts(z):
    import torch
    G = torch.zeros((4, 12), device="cuda")
    dO = torch.zeros((2, 4, 12), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((2, 4), device="cuda")
    L = z.lib()
    # d = 12 is not a multiple of 8 for bf16
    assert L.dust_attn_reward(G.data_ptr(), 12, dO.data_ptr(), 16, z.DUST_BF16, 4, 12, 2,
                              c.data_ptr(), 4, None) == z.DUST_ERR_UNSUPPORTED
    # misaligned ghat
    assert L.dust_attn_reward(G.data_ptr() + 4, 12, dO.data_ptr(), 16, z.DUST_F32, 4, 8, 2,
                              c.data_ptr(), 4, None) == z.DUST_ERR_INVALID_ARG
