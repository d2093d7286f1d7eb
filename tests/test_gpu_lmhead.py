"""LM-head perturbation on cached logits (Dust page, "간섭(interference) 줄이기"): the CUDA
cross-entropy loss change against the oracle, and the whole head estimate (credit, g on the
slab, slab rows of the head weight estimate) against the oracle chain.  Tolerances as for the
linear forward: the loss change is a short fp32 computation on exactly read inputs with
fp32 normals (element error <= 1e-3 x RMS, relative Frobenius <= 1e-4); g and G_W 2e-3."""
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


def _case(seed, N, V, dtype):
    import torch
    rng = np.random.default_rng(seed)
    logits = (rng.standard_normal((N, V)) * 2.0).astype(np.float32)
    y = rng.integers(0, V, size=N).astype(np.int32)
    if dtype == "bf16":
        bits = workloads.to_bf16_bits(logits)
        z64 = workloads.bf16_bits_to_f64(bits)
        zt = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        z64 = logits.astype(np.float64)
        zt = torch.from_numpy(logits).cuda()
    return zt, torch.from_numpy(y).cuda(), z64, y


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,V,v0,S,K,sigma", [
    (300, 512, 0, 512, 4, 1e-2),      # the whole vocabulary, series path
    (257, 1000, 128, 256, 3, 5e-2),   # a slab, expm1 path, ragged tokens
    (64, 4096, 1024, 1024, 2, 1e-3),
    (10, 96, 4, 20, 2, 1e-2),         # slab not a multiple of 16
    (50, 1002, 500, 500, 2, 1e-2),    # rows not a multiple of 16 bytes (bf16): scalar stats
])
def test_logits_ce_matches_oracle(z, dtype, N, V, v0, S, K, sigma):
    import torch
    zt, yt, z64, y = _case(N + V, N, V, dtype)
    key = z.NoiseKey(0x5EED0006, layer_id=48, draw_offset=5, token_offset=77)
    dl = z.dust_noisy_logits_ce(zt, yt, v0, S, K, sigma, key)
    torch.cuda.synchronize()
    loss, clean = oracle.noisy_logits_ce(z64, y, v0, S, K, sigma, key.seed, 48, 5, 77)
    _dev.assert_fp32_close(_dev.host(dl), loss - clean, "lm-head dloss")


def test_logits_ce_targets_outside_the_slab_and_invalid(z):
    import torch
    zt, yt, z64, y = _case(3, 40, 256, "f32")
    y[:20] = 5           # outside the slab [64, 192)
    y[20:] = 100         # inside
    yt = torch.from_numpy(y).cuda()
    dl = z.dust_noisy_logits_ce(zt, yt, 64, 128, 3, 1e-2, z.NoiseKey(9))
    torch.cuda.synchronize()
    loss, clean = oracle.noisy_logits_ce(z64, y, 64, 128, 3, 1e-2, 9)
    _dev.assert_fp32_close(_dev.host(dl), loss - clean, "targets in/out")
    y[7] = 256           # not a vocabulary index: NaN for that token only
    dl = z.dust_noisy_logits_ce(zt, torch.from_numpy(y).cuda(), 64, 128, 3, 1e-2, z.NoiseKey(9))
    h = _dev.host(dl)
    assert np.isnan(h[:, 7]).all() and np.isfinite(np.delete(h, 7, axis=1)).all()


def test_lm_head_estimate_matches_oracle_chain(z):
    """Cross-entropy loss change -> credit (gamma = 0: the head only changes its own token's
    loss) -> g on the slab and the slab's rows of the head weight estimate G_W = sum g h^T."""
    import torch
    N, V, d_model, v0, S, K, sigma = 512, 1024, 64, 256, 256, 8, 1e-2
    zt, yt, z64, y = _case(11, N, V, "bf16")
    H = workloads.custom_layer(12, N, d_model, 16, "bf16", 0.02)   # hidden states x = h
    h = _dev.to_device(H.x_store, "bf16")
    key = z.NoiseKey(0x5EED0006, layer_id=48)
    cu = np.array([0, N], dtype=np.int32)
    dl = z.dust_noisy_logits_ce(zt, yt, v0, S, K, sigma, key)
    r = z.dust_credit(dl, _dev.cu_to_device(cu), 0.0)
    GW, g = z.dust_weight_grad(r, h, S, K, sigma, key._replace(channel_offset=v0), g_out=True)
    torch.cuda.synchronize()
    loss, clean = oracle.noisy_logits_ce(z64, y, v0, S, K, sigma, key.seed, 48)
    r_ref = oracle.credit(loss, cu, 0.0)
    g_ref = oracle.output_error(r_ref, K, sigma, key.seed, V, 48, chans=np.arange(v0, v0 + S))
    GW_ref = oracle.weight_grad(g_ref, H.x_f64)
    assert _dev.rel_fro(_dev.host(g), g_ref) <= _dev.GW_FRO
    assert _dev.rel_fro(_dev.host(GW), GW_ref) <= _dev.GW_FRO


def test_head_workload_full_size_sampled(z):
    """The benchmarked head workload (16k tokens, vocabulary 4096, slab of 1024, K = 256) in
    the bench's launch configuration.  The oracle computes blocks of sampled tokens one by one
    (gamma = 0, so a token's credit needs only its own draws): loss change, credit and g on
    every slab channel.  G_W is checked through its definition against the GPU's own fp32 g
    (the sampled rows of which are pinned above), with the bf16 rounding bound of g."""
    import torch
    hw = workloads.HEAD_WORKLOADS["head-4096-slab1024"]
    data = workloads.generate_head(hw)
    zt = _dev.to_device(data.z_store, hw.dtype)
    h = _dev.to_device(data.h_store, hw.dtype)
    y = torch.from_numpy(data.y).cuda()
    cu = _dev.cu_to_device(data.cu_seqlens)
    key = z.NoiseKey(hw.seed, 48)
    dl = z.dust_noisy_logits_ce(zt, y, hw.v0, hw.S, hw.K, hw.sigma, key)
    r = z.dust_credit(dl, cu, hw.gamma)
    GW, g = z.dust_weight_grad(r, h, hw.S, hw.K, hw.sigma, key._replace(channel_offset=hw.v0),
                               g_out=True)
    torch.cuda.synchronize()
    assert z.dust_last_device_error()[0] == 0
    dl_h, r_h, g_h = _dev.host(dl), _dev.host(r), _dev.host(g)
    chans = np.arange(hw.v0, hw.v0 + hw.S)
    for t0 in (0, 2047, 9000, hw.N - 8):          # sequence starts, a boundary, the tail
        idx = np.arange(t0, t0 + 8)
        loss, clean = oracle.noisy_logits_ce(data.z_f64, data.y, hw.v0, hw.S, hw.K, hw.sigma,
                                             hw.seed, 48, tokens=idx)
        _dev.assert_fp32_close(dl_h[:, idx], loss - clean, f"dloss @{t0}")
        rr = oracle.credit(loss, np.array([0, 8], dtype=np.int32), hw.gamma)
        _dev.assert_fp32_close(r_h[:, idx], rr, f"r @{t0}")
        gr = oracle.output_error(rr, hw.K, hw.sigma, hw.seed, hw.V, 48, token_offset=t0,
                                 chans=chans)
        _dev.assert_fp32_close(g_h[idx], gr, f"g @{t0}")
    g64 = g.double()
    ref = (g64.t() @ h.double()).cpu().numpy()
    assert _dev.rel_fro(_dev.host(GW), ref) <= _dev.GW_FRO


def test_empty_slab_gives_zero_change_and_bad_slabs_are_rejected(z):
    """S = 0: no logit is perturbed, so every draw's loss change is exactly 0 (the oracle's
    special case); slabs that are not quad-aligned or leave the vocabulary are refused."""
    import torch
    zt, yt, z64, y = _case(5, 33, 64, "f32")
    dl = z.dust_noisy_logits_ce(zt, yt, 16, 0, 3, 1e-2, z.NoiseKey(4))
    torch.cuda.synchronize()
    assert np.array_equal(_dev.host(dl), np.zeros((3, 33), dtype=np.float32))
    loss, clean = oracle.noisy_logits_ce(z64, y, 16, 0, 3, 1e-2, 4)
    assert np.array_equal(loss - clean, np.zeros((3, 33)))
    for v0, S in ((2, 8), (0, 6), (60, 8)):
        with pytest.raises(z.DustError):
            z.dust_noisy_logits_ce(zt, yt, v0, S, 3, 1e-2, z.NoiseKey(4))
