"""The multi-GPU path's host logic with two gloo ranks on CPU.

Each rank takes whole sequences of one packed batch, computes its shard's estimate with
the global token offset (the oracle stands in for the kernels here), and the ranks sum the
weight estimates with an all-reduce.  The sum must equal the whole-batch estimate.  Failure
cases are made on the host: ranks that disagree on the problem, and a rank that leaves
before the collective.
"""
import os
import socket

import numpy as np
import pytest

from zeroth_order_transformer_b200 import distributed as zd


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_shard_by_sequences_whole_sequences_and_balance():
    import workloads
    cu = workloads.random_segments(5, 10000, 100, 900)
    for world in (1, 2, 3, 4, 8):
        shards = zd.shard_by_sequences(cu, world)
        assert shards[0][0] == 0 and shards[-1][1] == 10000
        for (a, b), (c, d) in zip(shards, shards[1:]):
            assert b == c
        for a, b in shards:
            assert a in cu and b in cu          # cuts fall on sequence ends
        sizes = [b - a for a, b in shards]
        assert max(sizes) - min(sizes) <= 2 * 900
    # fewer sequences than ranks: some shards are empty, none overlaps
    shards = zd.shard_by_sequences([0, 10, 20], 4)
    assert sum(b - a for a, b in shards) == 20
    t0, t1, local = zd.local_problem([0, 10, 25, 40], 2, 1)
    assert (t0, t1) == (25, 40) and list(local) == [0, 15]
    with pytest.raises(ValueError):
        zd.shard_by_sequences([0, 5, 3], 2)


def _worker(rank, world, port, mode, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=20))
    try:
        import oracle
        import workloads
        L = workloads.custom_layer(21, 600, 12, 16, "f32", None)
        cu = workloads.random_segments(22, 600, 40, 200)
        K, sigma, gamma, seed = 6, 1e-2, 0.9, 0x5EED0009
        if mode == "spsa":
            # weight-space probes: each rank's tokens give partial p; one all-reduce of P
            # scalars makes every rank's estimate the whole batch's
            Lb = workloads.custom_layer(31, 90, 8, 8, "bf16", 0.05)
            t0, t1 = (0, 40) if rank == 0 else (40, 90)
            pp, _, _ = oracle.spsa_probe(Lb.x_f64[t0:t1], Lb.W_f64, Lb.u_f64[t0:t1], 5, 1e-3,
                                         seed, 2)
            pt = torch.from_numpy(pp.copy())
            zd.allreduce_probe_scalars(pt)
            whole, _, _ = oracle.spsa_probe(Lb.x_f64, Lb.W_f64, Lb.u_f64, 5, 1e-3, seed, 2)
            G = oracle.spsa_estimate(pt.numpy(), 5, 8, 8, seed, 2)
            Gw = oracle.spsa_estimate(whole, 5, 8, 8, seed, 2)
            q.put((rank, float(max(np.abs(pt.numpy() - whole).max() / np.abs(whole).max(),
                                   np.linalg.norm(G - Gw) / np.linalg.norm(Gw)))))
            return
        if mode == "stack":
            # a stack of layers of different shapes: each rank's partial weight estimates
            # go into one flat buffer, summed over ranks in buckets of consecutive layers
            shapes = [(12, 16), (16, 8), (8, 24), (24, 12), (12, 12)]   # (d_in, d_out)
            lays = [workloads.custom_layer(40 + l, 600, di, do, "f32", None, layer_id=l)
                    for l, (di, do) in enumerate(shapes)]
            layout, total = zd.flat_layout([(do, di) for di, do in shapes])
            t0, t1, cu_local = zd.local_problem(cu, world, rank)
            flat = torch.zeros(total, dtype=torch.float64)
            for l, Ll in enumerate(lays):
                res = oracle.dust_layer(Ll.x_f64[t0:t1], Ll.W_f64, Ll.u_f64[t0:t1], K, sigma,
                                        gamma, cu_local, seed, layer_id=l, token_offset=t0)
                o, m = layout[l]
                flat[o:o + m] = torch.from_numpy(res["G_W"].reshape(-1))
            plan = zd.plan_buckets([m for _, m in layout], 3)
            covered = [l for a, b in plan for l in range(a, b)]
            assert covered == list(range(len(lays))), plan
            for bucket in plan:
                zd.allreduce_bucket(flat, layout, bucket)
            err = 0.0
            for l, Ll in enumerate(lays):
                whole = oracle.dust_layer(Ll.x_f64, Ll.W_f64, Ll.u_f64, K, sigma, gamma, cu, seed,
                                          layer_id=l)["G_W"]
                o, m = layout[l]
                got = flat[o:o + m].numpy().reshape(whole.shape)
                err = max(err, float(np.linalg.norm(got - whole) / np.linalg.norm(whole)))
            q.put((rank, err))
            return
        if mode == "mismatch":
            try:
                zd.check_same_problem(seed=seed + rank, K=K)
                q.put((rank, "no error"))
            except RuntimeError:
                q.put((rank, "raised"))
            return
        zd.check_same_problem(seed=seed, K=K, sigma=sigma, gamma=gamma, d_in=12, d_out=16)
        if mode == "dead" and rank == 1:
            q.put((rank, "left"))
            q.close()
            q.join_thread()                   # flush the message before leaving
            os._exit(0)                       # leaves between steps, before the collective
        t0, t1, cu_local = zd.local_problem(cu, world, rank)
        res = oracle.dust_layer(L.x_f64[t0:t1], L.W_f64, L.u_f64[t0:t1], K, sigma, gamma,
                                cu_local, seed, token_offset=t0)
        G = torch.from_numpy(res["G_W"].copy())
        try:
            zd.allreduce_weight_estimate(G)
        except Exception as e:  # noqa: BLE001
            q.put((rank, "collective failed: " + type(e).__name__))
            return
        whole = oracle.dust_layer(L.x_f64, L.W_f64, L.u_f64, K, sigma, gamma, cu, seed)
        err = float(np.linalg.norm(G.numpy() - whole["G_W"]) / np.linalg.norm(whole["G_W"]))
        q.put((rank, err))
    finally:
        if mode != "dead":
            dist.destroy_process_group()


def _run(mode, world=2, timeout=120):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, v = q.get(timeout=timeout)
        out[r] = v
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return out


def test_two_ranks_sum_to_whole_batch_estimate():
    out = _run("ok")
    assert set(out) == {0, 1}
    for r, err in out.items():
        assert isinstance(err, float) and err < 1e-10, (r, err)


def test_ranks_that_disagree_on_the_problem_raise():
    out = _run("mismatch")
    assert out == {0: "raised", 1: "raised"}


def test_rank_leaving_before_the_collective_fails_the_others():
    out = _run("dead")
    assert out[1] == "left"
    assert isinstance(out[0], str) and out[0].startswith("collective failed"), out[0]


def test_flat_layout_and_bucket_plan():
    layout, total = zd.flat_layout([(2304, 768), (768, 768), (3072, 768), (768, 3072)] * 12)
    assert all(o % 64 == 0 for o, _ in layout)              # 256-byte aligned views
    assert all(a[0] + a[1] <= b[0] for a, b in zip(layout, layout[1:]))
    assert total >= layout[-1][0] + layout[-1][1]
    sizes = [m for _, m in layout]
    for nb in (1, 2, 3, 4, 7, 48, 100):
        plan = zd.plan_buckets(sizes, nb)
        assert [l for a, b in plan for l in range(a, b)] == list(range(48))
        assert len(plan) == min(nb, 48)
    per = [sum(sizes[a:b]) for a, b in zd.plan_buckets(sizes, 4)]
    assert max(per) <= 1.2 * sum(sizes) / 4                 # whole blocks: even buckets
    # the default of the stack's calls and of bench.py: twelve buckets, one transformer block each
    assert zd.plan_buckets(sizes, 12) == [(4 * k, 4 * k + 4) for k in range(12)]
    a, b = zd.bucket_span(layout, (12, 24))
    assert a == layout[12][0] and b == layout[23][0] + layout[23][1]
    assert zd.plan_buckets([], 3) == [] and zd.plan_buckets([5, 1], 9) == [(0, 1), (1, 2)]


def test_two_ranks_stack_bucketed_sum_equals_whole_batch():
    out = _run("stack")
    assert set(out) == {0, 1}
    for r, err in out.items():
        assert isinstance(err, float) and err < 1e-10, (r, err)


def test_two_ranks_spsa_exchange_only_probe_scalars():
    out = _run("spsa")
    assert set(out) == {0, 1}
    for r, err in out.items():
        assert isinstance(err, float) and err < 1e-9, (r, err)
