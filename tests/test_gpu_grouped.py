"""Grouped calls (several layers sharing one token batch, one launch per step) against the
single-layer calls and against the oracle."""
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


def _stack(N, d, seed):
    """Two blocks of {QKV d->3d, O d->d, W_in d->4d, W_out 4d->d} (layer ids 4b + j)."""
    rng = np.random.default_rng(seed)
    shapes = []
    for b in range(2):
        shapes += [workloads.LayerShape(d, 3 * d, 4 * b), workloads.LayerShape(d, d, 4 * b + 1),
                   workloads.LayerShape(d, 4 * d, 4 * b + 2), workloads.LayerShape(4 * d, d, 4 * b + 3)]
    return [workloads.make_layer(rng, s, N, "bf16", 0.02) for s in shapes]


@pytest.mark.parametrize("N", [700, 8192])
def test_grouped_equals_single_layer_calls(z, N):
    """Bit-identical loss changes, credit and g, and G_W within fp32 rounding, at a ragged and
    at the stack's token count."""
    import torch
    K, sigma, gamma, seed = 6, 1e-3, 0.9, 0x5EED0005
    layers = _stack(N, 64, 1)
    cu = workloads.random_segments(2, N, 50, 300)
    cu_d = _dev.cu_to_device(cu)
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K, want_g=True)
    st.estimate(cu_d, sigma, gamma, seed)
    torch.cuda.synchronize()
    for l, (x, W, u, lid) in enumerate(dev_layers):
        key = z.NoiseKey(seed, lid)
        dl = z.dust_noisy_linear_fwd(x, W, u, K, sigma, key)
        r = z.dust_credit(dl, cu_d, gamma)
        GW, g = z.dust_weight_grad(r, x, W.shape[0], K, sigma, key, g_out=True)
        torch.cuda.synchronize()
        assert torch.equal(st.dloss[l], dl), l
        assert torch.equal(st.r[l], r), l
        assert torch.equal(st.g[l], g), l
        assert _dev.rel_fro(_dev.host(st.G_W[l]), _dev.host(GW)) < 1e-6, l


def test_grouped_stack_matches_oracle(z):
    import torch
    N, K, sigma, gamma, seed = 520, 8, 1e-3, 0.99, 0x5EED0005
    layers = _stack(N, 32, 3)
    cu = workloads.random_segments(4, N, 64, 256)
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K, want_g=True)
    st.estimate(_dev.cu_to_device(cu), sigma, gamma, seed)
    torch.cuda.synchronize()
    for l, L in enumerate(layers):
        ref = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, K, sigma, gamma, cu, seed,
                                L.shape.layer_id)
        _dev.assert_fp32_close(_dev.host(st.dloss[l]), ref["loss"] - ref["clean"], f"dloss {l}")
        assert _dev.rel_fro(_dev.host(st.g[l]), ref["g"]) <= _dev.GW_FRO, l
        assert _dev.rel_fro(_dev.host(st.G_W[l]), ref["G_W"]) <= _dev.GW_FRO, l


def test_stack_bucketed_reduce_sees_every_layer_once(z):
    """The stack's weight estimate in buckets of consecutive layers, each bucket's span of the
    flat G_W buffer handed to a collective on a side stream (here a stand-in that doubles it on
    the current stream): every layer comes out doubled, once."""
    import torch
    N, K, sigma, gamma, seed = 640, 6, 1e-3, 0.9, 0x5EED0005
    layers = _stack(N, 64, 7)
    cu_d = _dev.cu_to_device(workloads.random_segments(8, N, 50, 300))
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K)
    ref = [g.clone() for g in st.estimate(cu_d, sigma, gamma, seed)]
    for buckets in (1, 3, 8):
        seen = []

        def reduce(G):
            seen.append(G.numel())
            G.mul_(2.0)

        st.estimate(cu_d, sigma, gamma, seed, reduce=reduce, buckets=buckets)
        torch.cuda.synchronize()
        assert sum(seen) == sum(m for _, m in st.layout) and len(seen) == min(buckets, 8)
        for l in range(len(layers)):
            assert _dev.rel_fro(_dev.host(st.G_W[l]), 2.0 * _dev.host(ref[l])) < 1e-6, (buckets, l)


def test_stack_estimate_from_host_matches_device_inputs(z):
    """The stack from pinned host inputs (uploaded in buckets of layers, each bucket's estimate
    overlapped with the next bucket's upload and its G_W copied back while later buckets run)
    gives the estimate of the device inputs."""
    import torch
    N, K, sigma, gamma, seed = 1024, 8, 1e-3, 0.99, 0x5EED0005
    layers = _stack(N, 32, 9)
    cu = workloads.random_segments(10, N, 60, 200)
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K)
    ref = [_dev.host(g).copy() for g in st.estimate(_dev.cu_to_device(cu), sigma, gamma, seed)]
    host = [tuple(t.cpu().pin_memory() for t in (x, W, u)) for x, W, u, _ in dev_layers]
    for x, W, u, _ in dev_layers:
        for t in (x, W, u):
            t.zero_()
    G = st.estimate_from_host(host, cu, sigma, gamma, seed, chunks=4).numpy()
    for l, (o, m) in enumerate(st.layout):
        assert _dev.rel_fro(G[o:o + m].reshape(ref[l].shape), ref[l]) < 1e-5, l


@pytest.mark.parametrize("g_terms", [1, 2])
def test_grouped_more_layers_than_one_launch_holds(z, g_terms):
    """70 small layers: every stage runs as two launches (64 layers is one launch's table).
    Each layer equals its single-layer calls: loss change, credit and g bit for bit, G_W
    within fp32 rounding, for either number of bf16 terms of g."""
    import torch
    N, K, sigma, gamma, seed = 256, 4, 1e-3, 0.9, 0x5EED0011
    rng = np.random.default_rng(71)
    shapes = [workloads.LayerShape(16 * (1 + l % 3), 16 * (1 + (l * 5) % 4), l) for l in range(70)]
    layers = [workloads.make_layer(rng, sh, N, "bf16", 0.05) for sh in shapes]
    cu = workloads.random_segments(72, N, 20, 120)
    cu_d = _dev.cu_to_device(cu)
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K, want_g=True, g_terms=g_terms)
    st.estimate(cu_d, sigma, gamma, seed)
    torch.cuda.synchronize()
    assert z.dust_last_device_error()[0] == 0
    for l in (0, 1, 33, 63, 64, 65, 69):
        x, W, u, lid = dev_layers[l]
        key = z.NoiseKey(seed, lid)
        dl = z.dust_noisy_linear_fwd(x, W, u, K, sigma, key)
        r = z.dust_credit(dl, cu_d, gamma)
        GW, g = z.dust_weight_grad(r, x, W.shape[0], K, sigma, key, g_out=True, g_terms=g_terms)
        torch.cuda.synchronize()
        assert torch.equal(st.dloss[l], dl), l
        assert torch.equal(st.r[l], r), l
        assert torch.equal(st.g[l], g), l
        assert _dev.rel_fro(_dev.host(st.G_W[l]), _dev.host(GW)) < 1e-6, l
    # and against the oracle for the first and the last layer
    for l in (0, 69):
        L = layers[l]
        ref = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, K, sigma, gamma, cu, seed, l)
        assert _dev.rel_fro(_dev.host(st.G_W[l]), ref["G_W"]) <= (
            _dev.GW_FRO if g_terms == 1 else _dev.FP32_FRO), l


def test_stack_estimate_from_host_with_bucketed_reduce(z):
    """The host-input path with a reduction per bucket of layers (a stand-in collective that
    doubles its span on the side stream) before each bucket is copied back."""
    import torch
    N, K, sigma, gamma, seed = 512, 6, 1e-3, 0.9, 0x5EED0005
    layers = _stack(N, 32, 13)
    cu = workloads.random_segments(14, N, 60, 200)
    dev_layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in layers]
    st = z.DustStack(dev_layers, K)
    ref = [_dev.host(g).copy() for g in st.estimate(_dev.cu_to_device(cu), sigma, gamma, seed)]
    host = [tuple(t.cpu().pin_memory() for t in (x, W, u)) for x, W, u, _ in dev_layers]
    seen = []

    def reduce(G):
        seen.append(G.numel())
        G.mul_(2.0)

    G = st.estimate_from_host(host, cu, sigma, gamma, seed, chunks=3, reduce=reduce).numpy()
    assert sum(seen) == sum(m for _, m in st.layout) and len(seen) == 3
    for l, (o, m) in enumerate(st.layout):
        assert _dev.rel_fro(G[o:o + m].reshape(ref[l].shape), 2.0 * ref[l]) < 1e-5, l


def test_grouped_rejects_bad_descriptors(z):
    import ctypes
    d = (z.dust_layer_desc * 1)()
    d[0].d_in, d[0].d_out = 64, 72          # not a multiple of 16
    key = z.NoiseKey(1).c()
    assert z.lib().dust_noisy_linear_fwd_grouped(d, 1, 256, 4, 1e-3, key, None, 0, None) == \
        z.DUST_ERR_UNSUPPORTED
    assert z.lib().dust_noisy_linear_fwd_grouped(d, 0, 256, 4, 1e-3, key, None, 0, None) == \
        z.DUST_ERR_INVALID_ARG
