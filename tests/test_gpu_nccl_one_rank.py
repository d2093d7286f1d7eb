"""The stack's bucketed weight-estimate exchange through a real NCCL process group of one rank
on this GPU.  A one-rank all-reduce leaves the data as it is, so the exchanged estimate must
equal the estimate without exchange: bit for bit with one bucket, and within fp32 rounding with
several (a bucket of fewer layers has fewer output tiles, so its weight estimate may split the
token sum differently, split-K).  What the test exercises is the mechanics: each
bucket's collective issued on the side stream after its weight estimate, and the caller's
stream joined to it before the step ends (device inputs and host inputs).  No rank waits for
another: the multi-rank sums are checked with gloo on CPU (tests/test_distributed_cpu.py)."""
import os
import socket

import pytest

import workloads
from tests import _dev

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_bucketed_all_reduce_through_nccl_one_rank():
    import datetime

    import torch
    import torch.distributed as dist
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import zeroth_order_transformer_b200 as z
    from zeroth_order_transformer_b200 import distributed as zd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60), device_id=dev)
    try:
        data = workloads.generate(5, n_layers=8)
        wl = data.wl
        layers = [(*_dev.layer_to_device(L), L.shape.layer_id) for L in data.layers]
        cu = _dev.cu_to_device(data.cu_seqlens)
        st = z.DustStack(layers, wl.K)
        ref = st.estimate(cu, wl.sigma, 0.9, wl.seed)
        ref = [g.clone() for g in ref]
        for buckets in (1, 4):
            st.G_W_flat.fill_(float("nan"))
            st.estimate(cu, wl.sigma, 0.9, wl.seed, reduce=zd.allreduce_weight_estimate,
                        buckets=buckets)
            torch.cuda.synchronize()
            for l in range(len(layers)):
                if buckets == 1:
                    assert torch.equal(st.G_W[l], ref[l]), (buckets, l)
                else:
                    e = _dev.rel_fro(_dev.host(st.G_W[l]), _dev.host(ref[l]))
                    assert e <= _dev.FP32_FRO, (buckets, l, e)
        host = [tuple(t.cpu().pin_memory() for t in (x, W, u)) for x, W, u, _ in layers]
        G = st.estimate_from_host(host, data.cu_seqlens, wl.sigma, 0.9, wl.seed, chunks=4,
                                  reduce=zd.allreduce_weight_estimate)
        for l, (o, m) in enumerate(st.layout):
            got = G[o:o + m].view(ref[l].shape)
            assert _dev.rel_fro(got.numpy(), _dev.host(ref[l])) <= _dev.FP32_FRO, l
        assert z.dust_last_device_error()[0] == 0
    finally:
        dist.destroy_process_group()
