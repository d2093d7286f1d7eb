"""Parity at the benchmarked sizes, in bench.py's launch configuration, against the oracle's
own chain (workloads 2-4 whole; the whole 48-layer stack in one grouped launch per step, as
benchmarked, at the headline discount 0.9; two of its twelve blocks, grouped, at the three
discounts of its sweep with the fp32 g kept).

For every workload the oracle evaluates the whole forward (every token, draw and channel),
its centred loss and its credit over the real segments.  Compared:
  * the loss change and the credit of every token and draw (fp32 closeness; the credit at the
    general-gamma bound of the scan);
  * the 8192-token GPT-2-small MLP layer: g of every token and channel and the whole weight
    estimate G_W = sum_t g_t x_t^T, both from the oracle's own g;
  * the larger workloads and the stack: g and the rows of G_W of sampled output channels
    (both ends of every tensor-core tile among them), from the oracle's g of those channels
    over every token.
Tolerances as in the other parity tests: fp32 closeness for the loss change and fp32 g,
2e-3 relative Frobenius for G_W (g enters the tensor cores rounded)."""
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


def _channels(d_out):
    """Sampled output channels: the first and last of the layer, both ends of tile boundaries
    (128 and 256 channels) and a spread of interior ones."""
    c = {0, 1, 2, 3, d_out - 4, d_out - 1}
    for b in (127, 128, 255, 256, 383, 384):
        if b < d_out:
            c.add(b)
    c.update(int(v) for v in np.linspace(5, d_out - 6, 12).astype(int))
    return np.array(sorted(c), dtype=np.int32)


def _credit_tol(r_ref, cu, gamma):
    L = int(np.max(np.diff(cu)))
    eff = min(L, 1.0 / (1.0 - gamma) if gamma < 1 else L) + 1
    return 2e-6 * eff * np.max(np.abs(r_ref)) + 1e-6


def _check_chain(L, cu, K, sigma, gamma, seed, dl, r, g, GW, loss=None, full_gw=False):
    """Compare the GPU's loss change, credit, fp32 g (None: not kept by the GPU run) and G_W
    with the oracle's chain; loss (the oracle's absolute losses and clean losses) may be passed
    in when it is reused."""
    lid, d_out = L.shape.layer_id, L.shape.d_out
    if loss is None:
        loss = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, K, sigma, seed, lid)
    lo, clean = loss
    _dev.assert_fp32_close(dl, lo - clean, f"dloss layer {lid}")
    r_ref = oracle.credit(lo, cu, gamma)
    err = np.abs(r - r_ref).max()
    assert err <= _credit_tol(r_ref, cu, gamma), (lid, gamma, err)
    if full_gw:
        g_ref = oracle.output_error(r_ref, K, sigma, seed, d_out, lid)
        _dev.assert_fp32_close(g, g_ref, f"g layer {lid}")
        G_ref = oracle.weight_grad(g_ref, L.x_f64)
        e = _dev.rel_fro(GW, G_ref)
        print(f"layer {lid}: G_W rel-Fro {e:.3e} (whole matrix)")
        assert e <= _dev.GW_FRO, e
        return
    ch = _channels(d_out)
    g_ref = oracle.output_error(r_ref, K, sigma, seed, d_out, lid, chans=ch)
    if g is not None:
        _dev.assert_fp32_close(g[:, ch], g_ref, f"g layer {lid} sampled channels")
    rows = oracle.weight_grad(g_ref, L.x_f64)
    e = _dev.rel_fro(GW[ch], rows)
    print(f"layer {lid} gamma {gamma}: G_W rel-Fro {e:.3e} over {ch.size} sampled rows")
    assert e <= _dev.GW_FRO, e


@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_single_layer_workload_against_oracle_chain(z, cfg):
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
    host = [_dev.host(t) for t in (dl, r, g, GW)]
    del x, W, u, dl, r, g, GW, ws
    torch.cuda.empty_cache()
    _check_chain(L, cu, wl.K, wl.sigma, wl.gamma, wl.seed, *host, full_gw=(cfg == 2))


_LOSS = {}


def test_grouped_stack_against_oracle_chain(z):
    """The 48-layer stack's shapes (QKV 768->2304, O 768->768, W_in 768->3072, W_out
    3072->768) for two blocks, one grouped launch per step as in the bench, at gamma 0, 0.9
    and 0.99; the oracle's losses of the checked layers are computed once."""
    import torch
    data = workloads.generate(5, n_layers=8)
    wl = data.wl
    layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
    st = z.DustStack(layers, wl.K, want_g=True)
    cu = data.cu_seqlens
    cu_d = _dev.cu_to_device(cu)
    for gamma in wl.gammas:
        st.estimate(cu_d, wl.sigma, gamma, wl.seed)
        torch.cuda.synchronize()
        assert z.dust_last_device_error()[0] == 0
        for l in (0, 3, 5):
            L = data.layers[l]
            if l not in _LOSS:
                _LOSS[l] = oracle.noisy_linear_loss(L.x_f64, L.W_f64, L.u_f64, wl.K, wl.sigma,
                                                    wl.seed, L.shape.layer_id)
            _check_chain(L, cu, wl.K, wl.sigma, gamma, wl.seed, _dev.host(st.dloss[l]),
                         _dev.host(st.r[l]), _dev.host(st.g[l]), _dev.host(st.G_W[l]),
                         loss=_LOSS[l])


@pytest.fixture(scope="module")
def stack5():
    return workloads.generate(5)


def test_whole_48_layer_stack_as_benchmarked_against_oracle_chain(z, stack5):
    """All 48 layers of the 12-block stack, one grouped launch per kernel, no fp32 g kept,
    gamma 0.9: the launch that bench.py times.  Checked against the oracle: the first block's
    four layers and the last block's four (every layer shape, both ends of the layer table)."""
    import torch
    data = stack5
    wl = data.wl
    assert len(data.layers) == 48
    layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
    st = z.DustStack(layers, wl.K)
    cu = data.cu_seqlens
    gamma = 0.9
    st.estimate(_dev.cu_to_device(cu), wl.sigma, gamma, wl.seed)
    torch.cuda.synchronize()
    assert z.dust_last_device_error()[0] == 0
    checked = (0, 1, 2, 3, 44, 45, 46, 47)
    host = {l: (_dev.host(st.dloss[l]), _dev.host(st.r[l]), _dev.host(st.G_W[l]))
            for l in checked}
    del layers, st
    torch.cuda.empty_cache()
    for l in checked:
        dl, r, GW = host[l]
        _check_chain(data.layers[l], cu, wl.K, wl.sigma, gamma, wl.seed, dl, r, None, GW)


def test_whole_48_layer_stack_from_host_inputs_as_benchmarked(z, stack5):
    """The end-to-end form that bench.py times: the 48 layers' inputs in pinned host memory,
    uploaded in the default buckets of layers, each bucket estimated while the next one is
    uploaded, G_W read back bucket by bucket.  Every layer's G_W equals the estimate of the
    same inputs already on the device (fp32 rounding of the split-K sums, whose plan depends
    on the launch's tiles)."""
    import torch
    data = stack5
    wl = data.wl
    layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
    st = z.DustStack(layers, wl.K)
    cu = data.cu_seqlens
    ref = [_dev.host(g).copy() for g in st.estimate(_dev.cu_to_device(cu), wl.sigma, 0.9, wl.seed)]
    host = [tuple(t.cpu().pin_memory() for t in (x, W, u)) for x, W, u, _ in layers]
    for x, W, u, _ in layers:
        for t in (x, W, u):
            t.zero_()
    G = st.estimate_from_host(host, cu, wl.sigma, 0.9, wl.seed).numpy()
    assert z.dust_last_device_error()[0] == 0
    for l, (o, m) in enumerate(st.layout):
        e = _dev.rel_fro(G[o:o + m].reshape(ref[l].shape), ref[l])
        assert e < 1e-5, (l, e)
