"""Helpers shared by the GPU tests: move seeded inputs to the device, compare against the
oracle.  Imports torch lazily so the CPU suite can collect without a GPU."""
import numpy as np


def torch():
    import torch as _t
    return _t


def to_device(store: np.ndarray, dtype: str, device="cuda"):
    """A workloads ``*_store`` array (float32, or bf16 bits as uint16) as a device tensor."""
    t = torch()
    if dtype == "f32":
        return t.from_numpy(np.ascontiguousarray(store)).to(device)
    bits = t.from_numpy(np.ascontiguousarray(store).view(np.int16))
    return bits.view(t.bfloat16).to(device)


def layer_to_device(L, device="cuda"):
    return (to_device(L.x_store, L.dtype, device), to_device(L.W_store, L.dtype, device),
            to_device(L.u_store, L.dtype, device))


def cu_to_device(cu, device="cuda"):
    return torch().from_numpy(np.ascontiguousarray(cu, dtype=np.int32)).to(device)


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def host(t) -> np.ndarray:
    return t.detach().cpu().numpy()


# Tolerances (derivations in the tests' docstrings):
#   normals: |z_gpu - z_exact| <= 1e-5 absolute.
#   loss change, g (fp32 output): element error <= 1e-3 x RMS of the reference; relative
#     Frobenius error <= 1e-4.
#   G_W with bf16 g operand, and g itself: relative Frobenius error <= 2e-3.
NORMAL_ATOL = 1e-5
FP32_ELEM_RTOL_RMS = 1e-3
FP32_FRO = 1e-4
GW_FRO = 2e-3


def assert_fp32_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    rms = np.sqrt(np.mean(ref * ref))
    err = np.max(np.abs(got - ref))
    assert err <= FP32_ELEM_RTOL_RMS * rms, (what, err, rms)
    assert rel_fro(got, ref) <= FP32_FRO, (what, rel_fro(got, ref))
