"""dust_credit_no_alloc: the credit entry point for callers that cannot allocate device memory.

Such callers (a plugin run by an engine that owns all device memory, a process under a fixed
memory budget) cannot provide a workspace, so this entry point keeps the look-back scratch in
a static 4 MiB device array of the library.  The test calls it through the C ABI twice in a
row, with different inputs, and checks each result against dust_credit, the entry point with
a caller workspace, within the credit tolerance of the parity tests.  This file is collected
last so that a run stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu


def _tol(r_ref, cu, gamma):
    # fp32 scan rounding bound used by the credit parity tests
    L = np.max(np.diff(cu))
    eff = min(L, 1.0 / (1.0 - gamma) if gamma < 1 else L) + 1
    return 2e-6 * eff * np.max(np.abs(r_ref), axis=1, keepdims=True) + 1e-6


def test_no_alloc_credit_matches_workspace_entry_point_twice():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as z
    lib = z.lib()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(16, 5000, 0.95, 1, 1200, 11), (32, 20000, 0.99, 256, 2048, 12)]
    for K, N, gamma, lo, hi, seed in cases:
        cu_np = workloads.random_segments(seed, N, lo, hi)
        loss = torch.from_numpy(workloads.gaussian_losses(seed + 100, K, N)).cuda()
        cu = torch.from_numpy(cu_np).cuda()
        r_ref = z.dust_credit(loss, cu, gamma)
        r_new = torch.full((K, N), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.dust_credit_no_alloc(ctypes.c_void_p(loss.data_ptr()), N, K, N,
                                      ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1,
                                      ctypes.c_float(gamma), ctypes.c_void_p(r_new.data_ptr()), N,
                                      ctypes.c_void_p(stream))
        assert st == z.DUST_OK, z.status_string(st)
        torch.cuda.synchronize()
        a, b = r_new.cpu().numpy(), r_ref.cpu().numpy()
        assert np.all(np.isfinite(a))
        assert np.all(np.abs(a - b) <= _tol(b, cu_np, gamma))
    assert z.dust_last_device_error()[0] == z.DUST_OK


def test_no_alloc_credit_rejects_sizes_beyond_the_static_scratch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as z
    K, N = 64, 4_000_000  # needs about 32 MB of scratch, above the 4 MiB array
    need = z.dust_workspace_size(z.DUST_OP_CREDIT, z.DUST_F32, N, 0, 0, K)
    assert need > (4 << 20)
    loss = torch.zeros(16, dtype=torch.float32, device="cuda")
    cu = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    st = z.lib().dust_credit_no_alloc(ctypes.c_void_p(loss.data_ptr()), N, K, N,
                                      ctypes.c_void_p(cu.data_ptr()), 1, ctypes.c_float(0.9),
                                      ctypes.c_void_p(loss.data_ptr()), N, None)
    assert st == z.DUST_ERR_WORKSPACE
