"""The estimator's calls inside a CUDA graph.

Every call enqueues kernels (and, for the credit scan, memsets of its look-back state) on the
caller's stream and allocates nothing, so a whole step can be captured once and replayed: the
arguments (pointers, sizes, tensor maps) are fixed at capture time, and a replay recomputes
the estimate from whatever the captured input buffers then hold.  Replays must equal eager
calls bit for bit (every kernel is deterministic)."""
import numpy as np
import pytest

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


def test_stack_step_replays_from_a_cuda_graph(z):
    import torch
    data = workloads.generate(5, n_layers=8)
    wl = data.wl
    layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
    cu = _dev.cu_to_device(data.cu_seqlens)
    st = z.DustStack(layers, wl.K)
    st.estimate(cu, wl.sigma, 0.9, wl.seed)          # first call: one-time set-up outside capture
    torch.cuda.synchronize()
    eager = st.G_W_flat.clone()
    g = torch.cuda.CUDAGraph()
    st.G_W_flat.zero_()
    with torch.cuda.graph(g):
        st.estimate(cu, wl.sigma, 0.9, wl.seed)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(st.G_W_flat, eager)
    # new inputs in the captured buffers: the replay estimates them
    x0 = layers[0][0]
    x0.copy_(torch.flip(x0, dims=[0]))
    g.replay()
    torch.cuda.synchronize()
    replayed = st.G_W_flat.clone()
    st.estimate(cu, wl.sigma, 0.9, wl.seed)
    torch.cuda.synchronize()
    assert torch.equal(replayed, st.G_W_flat)
    assert not torch.equal(replayed[: st.layout[0][1]], eager[: st.layout[0][1]])
    assert z.dust_last_device_error()[0] == 0


def test_single_layer_chain_replays_from_a_cuda_graph(z):
    import torch
    L = workloads.custom_layer(61, 4100, 256, 512, "bf16", 0.02)
    x, W, u = _dev.layer_to_device(L)
    cu = _dev.cu_to_device(workloads.random_segments(62, 4100, 100, 900))
    K, sigma, gamma = 8, 1e-3, 0.95
    layer = z.DustLayer(4100, 256, 512, K, torch.bfloat16, x.device)
    key = z.NoiseKey(0x5EED0031, 3)
    eager = layer.estimate(x, W, u, cu, sigma, gamma, key).clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.estimate(x, W, u, cu, sigma, gamma, key)
    for _ in range(3):
        layer.G_W.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.G_W, eager)
    assert z.dust_last_device_error()[0] == 0
