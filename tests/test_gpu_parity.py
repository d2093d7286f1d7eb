"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded inputs.

Tolerances, from the arithmetic:
  * Philox words and all integer/segment logic: bit-exact.
  * Normals: the kernels evaluate Box-Muller in fp32: the hardware base-2 logarithm (absolute
    error about 2^-22, replaced by an exact-input series for u > 1 - 2^-10), y * rsqrt(y)
    (2 ulp), the angle in one FMA (at most 3.5e-7 rad) and the hardware sine/cosine on
    [-pi, pi) (absolute error about 2^-21); with |z| <= 5.77 the bound is a few 1e-6, tested
    at 1e-5 absolute.
  * Loss change and fp32 g: sums of d_out (or K) terms in fp32 whose inputs carry the normal
    error above: element error <= 1e-3 x RMS, relative Frobenius error <= 1e-4.
  * G_W (bf16): g enters the tensor cores rounded to bf16 (relative rounding error up to 2^-9,
    RMS about 1.7e-3 for a noise-dominated g); the required bar is 2e-3 relative Frobenius,
    against the oracle's G_W built from the oracle's own fp64 g.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests import _dev

pytestmark = pytest.mark.gpu

z = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global z
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as zz
    zz.lib()
    z = zz
    yield
    st, info = z.dust_last_device_error()
    assert st == 0, (st, info)


# ------------------------------------------------------------------------- generator
def test_philox_words_bit_exact_and_normals_close():
    import torch
    rng = np.random.default_rng(100)
    n = 1 << 18
    ctr = rng.integers(0, 2**32, size=(n, 4), dtype=np.uint64).astype(np.uint32)
    ctr[: n // 4, 1:] &= np.uint32(0xFFFF)
    ctr[n // 4: n // 2] |= np.uint32(0x80000000)
    seed = 0x5EED0002
    words_ref, z_ref = oracle.philox_batch(ctr, seed)
    w, zn = z.dust_debug_philox(torch.from_numpy(ctr.view(np.int32)).cuda(), seed)
    assert np.array_equal(_dev.host(w).view(np.uint32), words_ref)
    err = np.abs(_dev.host(zn).astype(np.float64) - z_ref)
    print(f"max |z_gpu - z_exact| over {4 * n} normals: {err.max():.3e}")
    assert err.max() <= _dev.NORMAL_ATOL, err.max()


def test_philox_words_match_published_known_answers():
    """The device generator on the published Philox4x32-10 known-answer vectors."""
    import torch
    from tests.test_oracle_noise import kat_vectors
    for ctr, key, out in kat_vectors():
        seed = int(key[0]) | (int(key[1]) << 32)
        w, _ = z.dust_debug_philox(torch.from_numpy(ctr.reshape(1, 4).view(np.int32)).cuda(), seed)
        assert np.array_equal(_dev.host(w).view(np.uint32)[0], out), (ctr, key)


def test_philox_words_bit_exact_over_1e8_counters():
    """Words are integers: the device equals the oracle bit for bit over 2^27 (1.3e8) sampled
    counters in chunks of 2^24, each chunk with its own 64-bit seed: uniform random words (every
    counter word >= 2^31 in about half the blocks, all four in 1/16), counters shaped like the
    estimator's (small quad, token, draw and layer words), and all-high words."""
    import torch
    rng = np.random.default_rng(4242)
    chunk, n_chunks, total = 1 << 24, 8, 0
    for c in range(n_chunks):
        ctr = rng.integers(0, 2**32, size=(chunk, 4), dtype=np.uint64).astype(np.uint32)
        if c % 4 == 1:
            ctr &= np.array([0xFFF, 0xFFFFF, 0xFFFF, 0x3F], dtype=np.uint32)
        elif c % 4 == 2:
            ctr |= np.uint32(0x80000000)
        seed = int(rng.integers(0, 2**63, dtype=np.int64)) * 2 + c % 2
        ref, _ = oracle.philox_batch(ctr, seed, want_normals=False)
        w, _ = z.dust_debug_philox(torch.from_numpy(ctr.view(np.int32)).cuda(), seed)
        got = _dev.host(w).view(np.uint32)
        assert np.array_equal(got, ref), (c, int(np.count_nonzero(np.any(got != ref, axis=1))))
        total += chunk
        del w
    assert total >= 10**8


def test_normals_near_u_one_and_u_zero():
    """Words whose uniforms sit at the ends of (0, 1): rho -> 0 and rho -> 5.77."""
    import torch
    seed = 0x77
    rng = np.random.default_rng(101)
    ctr = rng.integers(0, 2**32, size=(1 << 16, 4), dtype=np.uint64).astype(np.uint32)
    words_ref, z_ref = oracle.philox_batch(ctr, seed)
    _, zn = z.dust_debug_philox(torch.from_numpy(ctr.view(np.int32)).cuda(), seed)
    zn = _dev.host(zn).astype(np.float64)
    u0 = ((words_ref[:, 0] >> 9).astype(np.float64) * 2 + 1) * 2.0**-24
    extreme = (u0 > 0.999) | (u0 < 0.001)
    assert extreme.sum() > 50
    err = np.abs(zn[extreme] - z_ref[extreme]).max()
    print(f"max error at u0 < 0.001 or u0 > 0.999: {err:.3e}")
    assert err <= _dev.NORMAL_ATOL


def test_philox_only_probe_xors_the_mapped_words():
    """dust_debug_word_sum (the Philox-only rate probe) XORs exactly the words of the
    estimator's counters: channel quad, token offset, draw and layer."""
    n, nb, c0 = 300, 13, 8
    key = z.NoiseKey(0x5EED0002, layer_id=9, draw_offset=5, token_offset=1000, channel_offset=c0)
    got = _dev.host(z.dust_debug_word_sum(key, n, nb)).view(np.uint32)
    q, t = np.meshgrid(np.arange(nb, dtype=np.uint32) + np.uint32(c0 // 4),
                       np.arange(n, dtype=np.uint32) + np.uint32(1000), indexing="ij")
    ctr = np.stack([q, t, np.full_like(q, 5), np.full_like(q, 9)], axis=-1).reshape(-1, 4)
    words, _ = oracle.philox_batch(ctr, 0x5EED0002, want_normals=False)
    ref = np.bitwise_xor.reduce(words.reshape(nb, n, 4), axis=(0, 2))
    assert np.array_equal(got, ref)


def test_generator_throughput_probe_sums_the_mapped_normals():
    """dust_debug_normal_sum (the generator-only rate probe) adds exactly the estimator's
    normals: token offset, draw offset, layer and channel offset all enter the counter."""
    n, nq, c0 = 300, 17, 8
    key = z.NoiseKey(0x5EED0002, layer_id=9, draw_offset=5, token_offset=1000, channel_offset=c0)
    got = _dev.host(z.dust_debug_normal_sum(key, n, nq)).astype(np.float64)
    a = oracle.noise(key.seed, 9, n, c0 + 4 * nq, 1, draw_offset=5, token_offset=1000)
    ref = a[0, :, c0:].sum(axis=1)
    assert np.abs(got - ref).max() <= 4 * nq * _dev.NORMAL_ATOL


# ------------------------------------------------------------------------- forward
def _fwd_case(L, K, sigma, key):
    import torch
    x, W, u = _dev.layer_to_device(L)
    dl = z.dust_noisy_linear_fwd(x, W, u, K, sigma, key)
    torch.cuda.synchronize()
    loss, clean = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, K, sigma, key.seed,
                                           key.layer_id, key.draw_offset, key.token_offset)
    return _dev.host(dl), loss - clean


@pytest.mark.parametrize("N,d_in,d_out,K", [
    (128, 64, 256, 4),      # one tile
    (200, 64, 320, 5),      # ragged tokens and channels
    (385, 144, 528, 3),     # ragged everything, d_in not a multiple of 64
    (1, 16, 16, 2),         # smallest
    (700, 768, 512, 8),
])
def test_fwd_bf16_matches_oracle(N, d_in, d_out, K):
    L = workloads.custom_layer(1000 + N, N, d_in, d_out, "bf16", 0.02)
    key = z.NoiseKey(0x5EED0002, layer_id=3, draw_offset=7, token_offset=11)
    got, ref = _fwd_case(L, K, 1e-3, key)
    _dev.assert_fp32_close(got, ref, "dloss")


def test_fwd_bf16_both_forms_match_oracle():
    """Layers large enough for the one-tile-per-CTA form (three waves of two CTAs per SM) and
    just below it (the persistent form), with ragged token and channel tails."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for d_out, K in ((1040, 2), (784, 3)):
        n_t = -(-d_out // 256)
        for m_tiles, persistent in ((-(-6 * sms // n_t)), False), ((6 * sms - 1) // n_t, True):
            N = 128 * m_tiles - 37
            assert z.dust_debug_fwd_plan(N, K, [d_out], sms)[0] == persistent
            L = workloads.custom_layer(90 + N + d_out, N, 64, d_out, "bf16", 0.02)
            key = z.NoiseKey(0x5EED00B0 + K, layer_id=1, draw_offset=3, token_offset=5)
            got, ref = _fwd_case(L, K, 1e-3, key)
            _dev.assert_fp32_close(got, ref, f"dloss, persistent {persistent}, {N} x {d_out}")


def test_fwd_f32_tiny_workload_matches_oracle():
    data = workloads.generate(1)
    L = data.layers[0]
    wl = data.wl
    got, ref = _fwd_case(L, wl.K, wl.sigma, z.NoiseKey(wl.seed))
    _dev.assert_fp32_close(got, ref, "dloss f32")


def test_fwd_offsets_above_2_31():
    L = workloads.custom_layer(5, 130, 32, 48, "bf16", 0.02)
    key = z.NoiseKey(2**63 + 12345, layer_id=2**31 + 5, draw_offset=2**31 + 3,
                     token_offset=2**32 - 200)
    got, ref = _fwd_case(L, 3, 5e-3, key)
    _dev.assert_fp32_close(got, ref, "dloss offsets")


def test_fwd_deterministic():
    import torch
    L = workloads.custom_layer(6, 600, 256, 768, "bf16", 0.02)
    x, W, u = _dev.layer_to_device(L)
    key = z.NoiseKey(9)
    a = z.dust_noisy_linear_fwd(x, W, u, 6, 1e-3, key).clone()
    b = z.dust_noisy_linear_fwd(x, W, u, 6, 1e-3, key)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------------------------- credit
def _credit_gpu(loss_np, cu, gamma):
    import torch
    loss = torch.from_numpy(np.ascontiguousarray(loss_np, dtype=np.float32)).cuda()
    r = z.dust_credit(loss, _dev.cu_to_device(cu), gamma)
    torch.cuda.synchronize()
    return _dev.host(r)


CREDIT_SEGMENTS = {
    "single-tokens": lambda N: np.arange(N + 1, dtype=np.int32),
    "whole-stream": lambda N: np.array([0, N], dtype=np.int32),
    "straddling": lambda N: workloads.random_segments(31, N, 200, 700),
    "short": lambda N: workloads.random_segments(32, N, 1, 40),
    "packed-256-2048": lambda N: workloads.random_segments(33, N, 256, 2048),
}


@pytest.mark.parametrize("seg", list(CREDIT_SEGMENTS))
@pytest.mark.parametrize("gamma", [0.0, 1.0])
@pytest.mark.parametrize("K", [2, 8, 32, 128])
def test_credit_bit_exact_on_integer_losses(seg, gamma, K):
    """Integer losses in [-8, 8], K a power of two, segments <= 2048 tokens: every mean,
    centred loss and (for gamma in {0, 1}) every partial sum is a multiple of 1/K below 2^15,
    exact in fp32 in any order, so the GPU must equal the oracle bit for bit.  This pins the
    segment resets, the look-back chaining and all indexing."""
    N = 3000 if K <= 32 else 1500
    cu = CREDIT_SEGMENTS[seg](N)
    if seg == "whole-stream" and gamma == 1.0:
        cu = np.array([0, 1000, N], dtype=np.int32)  # keep every segment <= 2048
    loss = workloads.dyadic_losses(40 + K, K, N, scale_bits=0, max_abs=8)
    got = _credit_gpu(loss, cu, gamma)
    ref = oracle.credit(loss, cu, gamma)
    assert np.array_equal(got.astype(np.float64), ref), np.abs(got - ref).max()


@pytest.mark.parametrize("K", [2, 8])
def test_credit_bit_exact_past_the_aggregate_window(K):
    """Segments of 15k-25k tokens (look-back windows of more than 64 blocks, walked with
    inclusive values), gamma = 1, integer losses in [-8, 8]: every partial sum is a multiple of
    1/K below 2^19 (at most 25k tokens of |c| <= 16), exact in fp32 for K <= 8, so whichever
    inclusive value a block takes the credit equals the oracle's bit for bit."""
    N = 60000
    cu = workloads.random_segments(34, N, 15000, 25000)
    loss = workloads.dyadic_losses(50 + K, K, N, scale_bits=0, max_abs=8)
    got = _credit_gpu(loss, cu, 1.0)
    ref = oracle.credit(loss, cu, 1.0)
    assert np.array_equal(got.astype(np.float64), ref), np.abs(got - ref).max()
    assert z.dust_last_device_error()[0] == 0


def _credit_tol(ref_c, cu, gamma):
    """fp32 rounding bound of the reverse scan: each step rounds by 2^-24 relative and the
    rounding errors decay by gamma, so the error is below a few 2^-24 times the discounted sum
    of |r| (taken here as 1e-6 x (min(L, 1/(1-gamma)) + 1) x max|r| of the row) plus the
    centring's rounding."""
    K, N = ref_c.shape
    L = np.max(np.diff(cu))
    eff = min(L, 1.0 / (1.0 - gamma) if gamma < 1 else L) + 1
    return 2e-6 * eff * np.max(np.abs(ref_c), axis=1, keepdims=True) + 1e-6


@pytest.mark.parametrize("lo,hi", [(256, 2048), (4096, 4096), (7000, 8192)])
def test_credit_repeats_bit_for_bit_up_to_8192_token_segments(lo, hi):
    """With every segment at most 8192 tokens (64 look-back blocks) each block's carry is the
    fixed-order composition of the aggregates of its window, so repeated calls agree bit for
    bit, whatever the order in which the blocks ran (K = 64 x 1 Mi tokens, more blocks than
    the GPU holds at once)."""
    import torch
    K, N = 64, 1 << 20
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    loss = torch.randn((K, N), generator=g, device="cuda")
    cu = _dev.cu_to_device(workloads.random_segments(98, N, lo, hi))
    first = z.dust_credit(loss, cu, 0.99)
    for _ in range(4):
        again = z.dust_credit(loss, cu, 0.99)
        torch.cuda.synchronize()
        assert torch.equal(first, again)
    assert z.dust_last_device_error()[0] == 0


def test_credit_segments_longer_than_the_aggregate_window():
    """Segments of 20k to 60k tokens (windows past 64 blocks, walked with inclusive values):
    against the oracle within the scan's rounding bound."""
    N = 1 << 17
    cu = workloads.random_segments(97, N, 20000, 60000)
    loss = workloads.gaussian_losses(96, 8, N)
    got = _credit_gpu(loss, cu, 0.999)
    ref = oracle.credit(loss.astype(np.float64), cu, 0.999)
    assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, 0.999))
    assert z.dust_last_device_error()[0] == 0


@pytest.mark.parametrize("gamma", [0.5, 0.9, 0.95, 0.99])
def test_credit_general_gamma(gamma):
    K, N = 16, 5000
    cu = workloads.random_segments(50, N, 1, 1200)
    loss = workloads.gaussian_losses(51, K, N)
    got = _credit_gpu(loss, cu, gamma)
    ref = oracle.credit(loss, cu, gamma)
    assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, gamma))


def test_credit_ragged_and_minimal_sizes():
    for N, K in [(1, 2), (255, 3), (257, 5), (513, 64)]:
        cu = np.array([0, N], dtype=np.int32)
        loss = workloads.gaussian_losses(60 + N, K, N)
        got = _credit_gpu(loss, cu, 0.9)
        ref = oracle.credit(loss, cu, 0.9)
        assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, 0.9)), (N, K)


CREDIT_BLOCK = 128  # tokens per look-back block of the credit kernel


def test_credit_timeout_is_reported_and_context_survives():
    """A block that never publishes makes its predecessor's bounded wait run out: the call
    reports DUST_ERR_TIMEOUT, writes NaN there, and the next call is correct."""
    import torch
    B = CREDIT_BLOCK
    K, N = 4, B * 6
    cu = np.array([0, N], dtype=np.int32)
    loss = workloads.gaussian_losses(70, K, N)
    z.dust_debug_credit_skip_publish(3)
    r = z.dust_credit(torch.from_numpy(loss).cuda(), _dev.cu_to_device(cu), 0.9)
    st, info = z.dust_last_device_error()
    # block 2 waits for block 3; blocks 1 and 0 may look past block 2's aggregate and time
    # out on block 3 themselves, or receive block 2's NaN: either way they are NaN.
    assert st == z.DUST_ERR_TIMEOUT and 0 <= info <= 2, (st, info)
    rh = _dev.host(r)
    assert np.isnan(rh[:, :3 * B]).all()
    ref = oracle.credit(loss, cu, 0.9)
    tail = slice(3 * B, N)
    assert np.all(np.abs(rh[:, tail] - ref[:, tail]) <= _credit_tol(ref, cu, 0.9)[:, :1])
    got = _credit_gpu(loss, cu, 0.9)
    ref = oracle.credit(loss, cu, 0.9)
    assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, 0.9))
    assert z.dust_last_device_error()[0] == 0


@pytest.mark.parametrize("K", [129, 300])
def test_credit_many_draws_row_groups(K):
    """More than 128 draws: the per-token mean comes from a separate pass and the rows are
    scanned in groups with their own look-back chains."""
    N = 2000
    cu = workloads.random_segments(80, N, 100, 900)
    loss = workloads.dyadic_losses(81, K, N, scale_bits=0, max_abs=8)
    got = _credit_gpu(loss, cu, 1.0)
    ref = oracle.credit(loss, cu, 1.0)
    tol = 1e-6 * np.max(np.abs(ref)) + 1e-6   # mean over K not a power of two rounds
    assert np.abs(got - ref).max() <= tol
    g = workloads.gaussian_losses(82, K, N)
    got = _credit_gpu(g, cu, 0.95)
    ref = oracle.credit(g, cu, 0.95)
    assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, 0.95))


def test_credit_unaligned_leading_dimension():
    """Rows that do not start on 16 bytes (ld not a multiple of 4) take the plain-load path."""
    import torch
    K, N, ld = 8, 1001, 1003
    cu = workloads.random_segments(83, N, 50, 400)
    loss = workloads.gaussian_losses(84, K, N)
    buf = torch.zeros((K, ld), dtype=torch.float32, device="cuda")
    buf[:, :N] = torch.from_numpy(loss).cuda()
    out = torch.full((K, ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(z.dust_workspace_size(z.DUST_OP_CREDIT, z.DUST_F32, N, 0, 0, K),
                     dtype=torch.uint8, device="cuda")
    cu_d = _dev.cu_to_device(cu)
    st = z.lib().dust_credit(buf.data_ptr(), ld, K, N, cu_d.data_ptr(), len(cu) - 1,
                             0.9, out.data_ptr(), ld, ws.data_ptr(), ws.numel(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    got = _dev.host(out)[:, :N]
    ref = oracle.credit(loss, cu, 0.9)
    assert np.all(np.abs(got - ref) <= _credit_tol(ref, cu, 0.9))
    assert np.isnan(_dev.host(out)[:, N:]).all()     # nothing written past N


# ------------------------------------------------------------------------- weight estimate
def _wgrad_case(L, K_chunk, K_total, sigma, key, r_seed, dtype, g_terms=2):
    import torch
    N = L.x_store.shape[0]
    d_out = L.W_store.shape[0]
    r = workloads.gaussian_losses(r_seed, K_chunk, N, scale=0.05)
    x = _dev.to_device(L.x_store, dtype)
    GW, g = z.dust_weight_grad(torch.from_numpy(r).cuda(), x, d_out, K_total, sigma, key,
                               g_out=True, g_terms=g_terms)
    torch.cuda.synchronize()
    g_ref = oracle.output_error(r, K_total, sigma, key.seed, d_out, key.layer_id,
                                key.draw_offset, key.token_offset)
    GW_ref = oracle.weight_grad(g_ref, L.x_f64)
    return _dev.host(GW), _dev.host(g), GW_ref, g_ref


@pytest.mark.parametrize("g_terms", [1, 2])
@pytest.mark.parametrize("N,d_in,d_out,K", [
    (256, 256, 128, 4),
    (300, 272, 144, 6),      # ragged tokens, columns and rows
    (4100, 768, 512, 8),     # several token tiles: split-K
    (16, 16, 16, 2),
])
def test_weight_grad_bf16_matches_oracle(N, d_in, d_out, K, g_terms):
    """Random credit makes g pure noise, the worst case for the bf16 rounding of g: one term
    stays within the required 2e-3, two terms (hi + lo) within the fp32 bound 1e-4."""
    L = workloads.custom_layer(2000 + N, N, d_in, d_out, "bf16", 0.02)
    key = z.NoiseKey(0x5EED0003, layer_id=1, draw_offset=40, token_offset=3)
    GW, g, GW_ref, g_ref = _wgrad_case(L, K, K + 40, 1e-3, key, 80 + N, "bf16", g_terms)
    _dev.assert_fp32_close(g, g_ref, "g")
    e = _dev.rel_fro(GW, GW_ref)
    print(f"G_W rel-Fro with {g_terms} bf16 term(s) of g: {e:.3e}")
    assert e <= (_dev.GW_FRO if g_terms == 1 else _dev.FP32_FRO), e


def test_weight_grad_f32_matches_oracle():
    L = workloads.custom_layer(3, 128, 64, 64, "f32", None)
    key = z.NoiseKey(0x5EED0001)
    GW, g, GW_ref, g_ref = _wgrad_case(L, 8, 8, 1e-2, key, 90, "f32")
    _dev.assert_fp32_close(g, g_ref, "g f32")
    _dev.assert_fp32_close(GW, GW_ref, "G_W f32")


def test_weight_grad_f32_odd_quad_count_matches_oracle():
    # d_out = 36: nine channel quads per token, so the last thread of every row owns one quad
    L = workloads.custom_layer(4, 77, 40, 36, "f32", None)
    key = z.NoiseKey(0x5EED0004, layer_id=2, draw_offset=5, token_offset=9)
    GW, g, GW_ref, g_ref = _wgrad_case(L, 5, 7, 1e-2, key, 91, "f32")
    _dev.assert_fp32_close(g, g_ref, "g f32, odd quad count")
    _dev.assert_fp32_close(GW, GW_ref, "G_W f32, odd quad count")


def test_weight_grad_accumulates_draw_chunks():
    """Two chunks (draw offsets 0 and K1) with accumulate give the full-population G_W."""
    import torch
    N, d_in, d_out, K, K1 = 512, 128, 256, 12, 5
    L = workloads.custom_layer(7, N, d_in, d_out, "bf16", 0.02)
    x = _dev.to_device(L.x_store, "bf16")
    r = workloads.gaussian_losses(91, K, N, scale=0.05)
    rt = torch.from_numpy(r).cuda()
    key0 = z.NoiseKey(11, layer_id=4, draw_offset=0)
    key1 = z.NoiseKey(11, layer_id=4, draw_offset=K1)
    GW, _ = z.dust_weight_grad(rt[:K1].contiguous(), x, d_out, K, 1e-3, key0)
    z.dust_weight_grad(rt[K1:].contiguous(), x, d_out, K, 1e-3, key1, G_W=GW, accumulate=True)
    torch.cuda.synchronize()
    g_ref = oracle.output_error(r, K, 1e-3, 11, d_out, 4)
    assert _dev.rel_fro(_dev.host(GW), oracle.weight_grad(g_ref, L.x_f64)) <= _dev.GW_FRO


# ------------------------------------------------------------------------- whole chain
def _chain(L, cu, K, sigma, gamma, key, dtype):
    import torch
    x, W, u = (_dev.to_device(a, dtype) for a in (L.x_store, L.W_store, L.u_store))
    d_out = W.shape[0]
    dl = z.dust_noisy_linear_fwd(x, W, u, K, sigma, key)
    r = z.dust_credit(dl, _dev.cu_to_device(cu), gamma)
    GW, g = z.dust_weight_grad(r, x, d_out, K, sigma, key, g_out=True)
    torch.cuda.synchronize()
    return {k: _dev.host(v) for k, v in dict(dloss=dl, r=r, g=g, G_W=GW).items()}


@pytest.mark.parametrize("gamma", [0.9, 0.0])
def test_chain_tiny_f32_workload(gamma):
    data = workloads.generate(1)
    L, wl = data.layers[0], data.wl
    got = _chain(L, data.cu_seqlens, wl.K, wl.sigma, gamma, z.NoiseKey(wl.seed), "f32")
    ref = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, wl.K, wl.sigma, gamma, data.cu_seqlens,
                            wl.seed)
    _dev.assert_fp32_close(got["dloss"], ref["loss"] - ref["clean"], "dloss")
    _dev.assert_fp32_close(got["r"], ref["r"], "r")
    assert _dev.rel_fro(got["g"], ref["g"]) <= _dev.GW_FRO
    assert _dev.rel_fro(got["G_W"], ref["G_W"]) <= _dev.GW_FRO


def test_chain_bf16_ragged_packed():
    N, d_in, d_out, K = 1000, 160, 272, 8
    L = workloads.custom_layer(8, N, d_in, d_out, "bf16", 0.02)
    cu = workloads.random_segments(9, N, 50, 400)
    key = z.NoiseKey(0x5EED0003, layer_id=2)
    got = _chain(L, cu, K, 1e-3, 0.99, key, "bf16")
    ref = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, K, 1e-3, 0.99, cu, key.seed, 2)
    _dev.assert_fp32_close(got["dloss"], ref["loss"] - ref["clean"], "dloss")
    assert _dev.rel_fro(got["r"], ref["r"]) <= 1e-4
    assert _dev.rel_fro(got["g"], ref["g"]) <= _dev.GW_FRO
    assert _dev.rel_fro(got["G_W"], ref["G_W"]) <= _dev.GW_FRO
    # the credit sums to zero over draws at every token (centring), to fp32 rounding
    assert np.abs(got["r"].sum(axis=0)).max() <= 1e-4 * np.abs(got["r"]).max()


def test_estimate_from_host_pipelined_matches_oracle():
    """DustLayer.estimate_from_host: pinned host inputs uploaded in runs of whole sequences
    while earlier runs are estimated; the noise keeps the whole batch's token indices."""
    import torch
    N, d_in, d_out, K, sigma, gamma = 1000, 128, 256, 8, 1e-3, 0.9
    L = workloads.custom_layer(31, N, d_in, d_out, "bf16", 0.02)
    cu = np.array([0, 240, 500, 764, 1000], dtype=np.int32)
    key = z.NoiseKey(0x5EED00C1, layer_id=4, token_offset=77)

    def pinned(store):
        return torch.from_numpy(np.ascontiguousarray(store).view(np.int16)).view(
            torch.bfloat16).pin_memory()

    layer = z.DustLayer(N, d_in, d_out, K, torch.bfloat16, "cuda")
    G = layer.estimate_from_host(pinned(L.x_store), pinned(L.W_store), pinned(L.u_store), cu,
                                 sigma, gamma, key, chunks=3)
    ref = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, K, sigma, gamma, cu, key.seed, 4,
                            token_offset=77)
    _dev.assert_fp32_close(_dev.host(layer.dloss), ref["loss"] - ref["clean"], "dloss")
    assert _dev.rel_fro(_dev.host(layer.r), ref["r"]) <= 1e-4
    assert _dev.rel_fro(G.numpy(), ref["G_W"]) <= _dev.GW_FRO
