"""Parity at the benchmarked sizes, in bench.py's launch configuration, on sampled outputs the
oracle computes one by one (workloads 2-4 whole; the 48-layer stack's shapes with two of its
twelve blocks, grouped).

A sampled window starts at token t0 and runs to the end of t0's sequence or until
gamma^len <= 1e-10, whichever comes first; the oracle evaluates the window's losses, its
centred loss and credit (the window as one segment), and g of its first tokens, whose credit
then differs from the whole sequence's by at most gamma^(len - 8) max|c| / (1 - gamma).
Compared: the loss change of every token of the window, the credit and g of its first eight
tokens.  G_W is checked at full size through its definition, sum_t g_t x_t^T, with the GPU's
own fp32 g (whose sampled rows are pinned above) and the bf16 rounding bound.  Tolerances as
in the other parity tests (fp32 closeness for the loss change and the credit, 2e-3 for g and
G_W)."""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import _dev

pytestmark = pytest.mark.gpu

FIRST = 8


@pytest.fixture(scope="module")
def z():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as zz
    zz.lib()
    return zz


def _window(cu, t0, gamma):
    s = int(np.searchsorted(cu, t0, side="right")) - 1
    end = int(cu[s + 1])
    if gamma == 0.0:
        return t0, min(end, t0 + FIRST)
    w = int(math.ceil(math.log(1e-10) / math.log(gamma))) + FIRST
    return t0, min(end, t0 + w)


def _check_window(L, cu, K, sigma, gamma, seed, layer_id, dl, r, g, t0):
    a, b = _window(cu, t0, gamma)
    idx = np.arange(a, b)
    loss, clean = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, K, sigma, seed, layer_id,
                                           tokens=idx)
    _dev.assert_fp32_close(dl[:, a:b], loss - clean, f"dloss layer {layer_id} @{t0}")
    rw = oracle.credit(loss, np.array([0, b - a], dtype=np.int32), gamma)
    m = min(FIRST, b - a)
    ref = rw[:, :m]
    got = r[:, a:a + m]
    tol = 2e-6 * (min(b - a, 1.0 / max(1e-12, 1.0 - gamma)) + 1) * np.abs(rw).max() + 1e-6
    assert np.abs(got - ref).max() <= tol, (layer_id, t0, np.abs(got - ref).max(), tol)
    d_out = L.W_f64.shape[0]
    gw = oracle.output_error(ref, K, sigma, seed, d_out, layer_id, token_offset=a)
    assert _dev.rel_fro(g[a:a + m], gw) <= _dev.GW_FRO, (layer_id, t0)


def _check_gw(g, x_f64, GW):
    ref = g.astype(np.float64).T @ x_f64
    assert _dev.rel_fro(GW, ref) <= _dev.GW_FRO


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_single_layer_workload_sampled(z, cfg):
    import torch
    data = workloads.generate(cfg)
    wl = data.wl
    L = data.layers[0]
    x, W, u = _dev.layer_to_device(L)
    cu = data.cu_seqlens
    key = z.NoiseKey(wl.seed, L.shape.layer_id)
    ws = torch.empty(max(z.dust_workspace_size(op, 1, wl.N, L.shape.d_in, L.shape.d_out, wl.K)
                         for op in range(3)), dtype=torch.uint8, device="cuda")
    dl = z.dust_noisy_linear_fwd(x, W, u, wl.K, wl.sigma, key, workspace=ws)
    r = z.dust_credit(dl, _dev.cu_to_device(cu), wl.gamma, workspace=ws)
    GW, g = z.dust_weight_grad(r, x, L.shape.d_out, wl.K, wl.sigma, key, g_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert z.dust_last_device_error()[0] == 0
    dl_h, r_h, g_h = _dev.host(dl), _dev.host(r), _dev.host(g)
    seg_starts = [int(c) for c in cu[:-1]]
    samples = [0, seg_starts[len(seg_starts) // 2] + 37, int(cu[1]) - 5, wl.N - 3]
    for t0 in samples:
        _check_window(L, cu, wl.K, wl.sigma, wl.gamma, wl.seed, L.shape.layer_id, dl_h, r_h,
                      g_h, t0)
    _check_gw(g_h, L.x_f64, _dev.host(GW))


@pytest.mark.parametrize("gamma", [0.0, 0.99])
def test_grouped_stack_sampled(z, gamma):
    """The 48-layer stack's shapes (QKV 768->2304, O 768->768, W_in 768->3072, W_out
    3072->768) for two blocks, one grouped launch per step as in the bench."""
    import torch
    data = workloads.generate(5, n_layers=8)
    wl = data.wl
    layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
    st = z.DustStack(layers, wl.K, want_g=True)
    st.estimate(_dev.cu_to_device(data.cu_seqlens), wl.sigma, gamma, wl.seed)
    torch.cuda.synchronize()
    assert z.dust_last_device_error()[0] == 0
    cu = data.cu_seqlens
    for l in (0, 3, 5):
        L = data.layers[l]
        dl_h, r_h, g_h = _dev.host(st.dloss[l]), _dev.host(st.r[l]), _dev.host(st.g[l])
        for t0 in (11, 3000, wl.N - 9):
            _check_window(L, cu, wl.K, wl.sigma, gamma, wl.seed, L.shape.layer_id, dl_h, r_h,
                          g_h, t0)
        _check_gw(g_h, L.x_f64, _dev.host(st.G_W[l]))
