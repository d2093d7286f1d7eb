"""dust_credit_no_alloc: the credit entry point for callers that cannot allocate device memory.

Such callers (a plugin run by an engine that owns all device memory, a process under a fixed
memory budget) cannot provide a workspace, so this entry point keeps the look-back scratch in
a static 4 MiB device array of the library.  The tests call it through the C ABI:
  * twice in a row, with different inputs, each result checked against dust_credit (the entry
    point with a caller workspace) within the credit tolerance of the parity tests;
  * on integer losses with a power-of-two draw count, where every partial sum is exact in
    fp32, bit for bit against the oracle's credit;
  * with more than 128 draws (several row groups, whose per-token mean also lives in the
    static array), with row strides larger than N, and with a large call followed by a small
    one and the other way round (the small call must not read what the large one left);
  * through the Python binding, which must reject a mis-shaped result matrix.
This file is collected last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def z():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as zz
    zz.lib()
    return zz


def _tol(r_ref, cu, gamma):
    # fp32 scan rounding bound used by the credit parity tests
    L = np.max(np.diff(cu))
    eff = min(L, 1.0 / (1.0 - gamma) if gamma < 1 else L) + 1
    return 2e-6 * eff * np.max(np.abs(r_ref), axis=1, keepdims=True) + 1e-6


def _call(z, loss, ld_loss, K, N, cu, gamma, r, ld_r):
    """dust_credit_no_alloc through the C ABI on the current stream."""
    import torch
    stream = torch.cuda.current_stream().cuda_stream
    return z.lib().dust_credit_no_alloc(ctypes.c_void_p(loss.data_ptr()), ld_loss, K, N,
                                        ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1,
                                        ctypes.c_float(gamma), ctypes.c_void_p(r.data_ptr()),
                                        ld_r, ctypes.c_void_p(stream))


def _case(z, K, N, gamma, lo, hi, seed, ld_extra=0, losses=None):
    """(no-alloc result, workspace-entry result, cu) for one seeded case; ld = N + ld_extra."""
    import torch
    cu_np = workloads.random_segments(seed, N, lo, hi)
    vals = losses if losses is not None else workloads.gaussian_losses(seed + 100, K, N)
    ld = N + ld_extra
    loss_full = torch.full((K, ld), float("nan"), dtype=torch.float32, device="cuda")
    loss_full[:, :N] = torch.from_numpy(vals).cuda()
    loss = loss_full[:, :N]
    cu = torch.from_numpy(cu_np).cuda()
    r_ref = z.dust_credit(loss, cu, gamma)
    r_full = torch.full((K, ld), float("nan"), dtype=torch.float32, device="cuda")
    st = _call(z, loss_full, ld, K, N, cu, gamma, r_full, ld)
    assert st == z.DUST_OK, z.status_string(st)
    torch.cuda.synchronize()
    out = r_full.cpu().numpy()
    assert np.all(np.isnan(out[:, N:]))           # nothing written past N in a row
    return out[:, :N], r_ref.cpu().numpy(), cu_np


def test_no_alloc_credit_matches_workspace_entry_point_twice(z):
    for K, N, gamma, lo, hi, seed in [(16, 5000, 0.95, 1, 1200, 11), (32, 20000, 0.99, 256, 2048, 12)]:
        a, b, cu = _case(z, K, N, gamma, lo, hi, seed)
        assert np.all(np.isfinite(a))
        assert np.all(np.abs(a - b) <= _tol(b, cu, gamma))
    assert z.dust_last_device_error()[0] == z.DUST_OK


def test_no_alloc_credit_bit_exact_against_oracle_on_dyadic_losses(z):
    """Integer losses in [-8, 8] with K a power of two <= 128, gamma in {0, 1} and segments of
    at most 2048 tokens: every mean, centred value and partial sum is a multiple of 1/K below
    2^15, exact in fp32, so the result must equal the oracle's credit bit for bit."""
    for K, N, gamma, lo, hi, seed in [(8, 3000, 1.0, 1, 700, 21), (64, 9000, 0.0, 100, 2048, 22),
                                      (128, 4100, 1.0, 200, 1500, 23)]:
        losses = workloads.dyadic_losses(seed, K, N, scale_bits=0, max_abs=8)
        a, _, cu = _case(z, K, N, gamma, lo, hi, seed, losses=losses)
        ref = oracle.credit(losses.astype(np.float64), cu, gamma)
        assert np.array_equal(a.astype(np.float64), ref), (K, N, gamma)


def test_no_alloc_credit_many_draws_and_row_strides(z):
    """K = 160 (two row groups plus the per-token mean in the static array) and row strides
    larger than N, against dust_credit and the oracle."""
    for K, N, gamma, ld_extra, seed in [(160, 6000, 0.9, 0, 31), (24, 7001, 0.95, 36, 32),
                                        (160, 3000, 0.99, 12, 33)]:
        a, b, cu = _case(z, K, N, gamma, 50, 1500, seed, ld_extra=ld_extra)
        assert np.all(np.abs(a - b) <= _tol(b, cu, gamma)), (K, N)
        ref = oracle.credit(workloads.gaussian_losses(seed + 100, K, N).astype(np.float64), cu,
                            gamma)
        assert np.all(np.abs(a - ref) <= _tol(ref, cu, gamma)), (K, N)
    assert z.dust_last_device_error()[0] == z.DUST_OK


def test_no_alloc_credit_large_then_small_and_small_then_large(z):
    """The array keeps the previous call's contents: a small call after a large one (and the
    reverse) must give the workspace entry point's result."""
    big = (64, 500000, 0.99, 256, 2048, 41)
    small = (16, 3000, 0.9, 64, 900, 42)
    for order in ((big, small), (small, big)):
        for K, N, gamma, lo, hi, seed in order:
            a, b, cu = _case(z, K, N, gamma, lo, hi, seed)
            assert np.all(np.abs(a - b) <= _tol(b, cu, gamma)), (K, N)
    assert z.dust_last_device_error()[0] == z.DUST_OK


def test_no_alloc_python_binding_checks_shapes(z):
    import torch
    K, N = 8, 1000
    cu_np = workloads.random_segments(51, N, 50, 400)
    cu = torch.from_numpy(cu_np).cuda()
    base = torch.from_numpy(workloads.gaussian_losses(52, K, N + 20)).cuda()
    loss = base[:, :N]                             # row-strided view
    r = torch.empty((K, N), dtype=torch.float32, device="cuda")
    z.dust_credit_no_alloc(loss, cu, 0.9, r)
    ref = z.dust_credit(loss, cu, 0.9)
    torch.cuda.synchronize()
    assert torch.equal(r, ref)
    with pytest.raises(ValueError):
        z.dust_credit_no_alloc(loss, cu, 0.9, torch.empty((K, N - 4), device="cuda"))
    with pytest.raises(ValueError):
        z.dust_credit_no_alloc(loss, cu, 0.9, torch.empty((K - 1, N), device="cuda"))
    with pytest.raises(TypeError):
        z.dust_credit_no_alloc(loss, cu, 0.9, torch.empty((K, N), dtype=torch.float64,
                                                          device="cuda"))


def test_no_alloc_credit_rejects_sizes_beyond_the_static_scratch(z):
    import torch
    for K, N in [(64, 4_000_000), (32, 1_048_448 + 128), (256, 116_480 + 128)]:
        need = z.dust_workspace_size(z.DUST_OP_CREDIT, z.DUST_F32, N, 0, 0, K)
        assert need > (4 << 20)
        loss = torch.zeros(16, dtype=torch.float32, device="cuda")
        cu = torch.tensor([0, N], dtype=torch.int32, device="cuda")
        st = z.lib().dust_credit_no_alloc(ctypes.c_void_p(loss.data_ptr()), N, K, N,
                                          ctypes.c_void_p(cu.data_ptr()), 1, ctypes.c_float(0.9),
                                          ctypes.c_void_p(loss.data_ptr()), N, None)
        assert st == z.DUST_ERR_WORKSPACE
    # the largest accepted sizes fit exactly
    for K, N in [(32, 1_048_448), (256, 116_480)]:
        assert z.dust_workspace_size(z.DUST_OP_CREDIT, z.DUST_F32, N, 0, 0, K) <= (4 << 20)
