"""Data-parallel plumbing for the Dust estimator across GPUs (one process per GPU).

The estimator shards by tokens.  Each rank takes whole sequences (the credit scan never
crosses a sequence end), generates the noise of its tokens with their GLOBAL index
(token_offset), so no noise and no loss is ever exchanged.  The only exchange is the sum
of the partial weight estimates G_W over ranks: one all-reduce per layer, or, for a stack of
layers, one per bucket of consecutive layers issued while the later buckets are still being
estimated.  This follows the
pages' remark that zeroth-order training needs to share only seeds and scalars
(gist.science 2605.15622, seed-based communication; gist.science 2502.10239, seed and scalar
upload), and the weight-estimate equation of the Dust page (G_W = sum over ALL tokens).

Nothing here computes any step of the estimator; `estimate_sharded` calls the CUDA path.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def shard_by_sequences(cu_seqlens: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Contiguous token ranges [t0, t1), one per rank, made of whole sequences, with token
    counts as even as the sequence boundaries allow (greedy on the ideal cut points).
    Ranks may receive an empty range when there are fewer sequences than ranks."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if cu.ndim != 1 or cu.size < 2 or cu[0] != 0 or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must be non-decreasing, start at 0, have >= 2 entries")
    if world < 1:
        raise ValueError("world must be >= 1")
    N = int(cu[-1])
    cuts = [0]
    for r in range(1, world):
        ideal = r * N / world
        j = int(np.argmin(np.abs(cu - ideal)))
        cuts.append(max(int(cu[j]), cuts[-1]))
    cuts.append(N)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def local_problem(cu_seqlens: Sequence[int], world: int, rank: int):
    """(t0, t1, local cu_seqlens as int32) of this rank's shard."""
    t0, t1 = shard_by_sequences(cu_seqlens, world)[rank]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    inside = cu[(cu > t0) & (cu < t1)]
    local = np.concatenate([[0], inside - t0, [t1 - t0]]).astype(np.int32)
    if t1 == t0:
        local = np.zeros(1, dtype=np.int32)
    return t0, t1, local


def check_same_problem(group=None, **fields) -> None:
    """Raise on every rank if the ranks disagree on any field (seed, K, sigma, gamma, layer,
    shapes): a mismatch would silently combine estimates of different problems."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    mine = tuple(sorted(fields.items()))
    everyone = [None] * world
    dist.all_gather_object(everyone, mine, group=group)
    bad = [r for r, v in enumerate(everyone) if v != mine]
    if bad:
        raise RuntimeError(f"ranks {bad} disagree on the estimator problem: {everyone}")


def allreduce_weight_estimate(G_W, group=None):
    """Sum of the per-rank partial weight estimates (in place)."""
    import torch.distributed as dist
    dist.all_reduce(G_W, op=dist.ReduceOp.SUM, group=group)
    return G_W


def flat_layout(shapes: Sequence[Tuple[int, int]], align: int = 64):
    """Where each layer's weight estimate G_W [d_out, d_in] sits in one flat fp32 buffer:
    ([(offset, size)] per layer, total elements).  Offsets are multiples of ``align`` elements
    (256 bytes), so every layer's view is aligned for the kernels and a bucket of consecutive
    layers is one contiguous span for one collective."""
    out, o = [], 0
    for d_out, d_in in shapes:
        n = int(d_out) * int(d_in)
        out.append((o, n))
        o += -(-n // align) * align
    return out, o


def plan_buckets(sizes: Sequence[int], n_buckets: int) -> List[Tuple[int, int]]:
    """Consecutive layer ranges [l0, l1) with element counts as even as the layer boundaries
    allow (cut where the running total is nearest k/n_buckets of the whole).  Every range is
    non-empty; fewer ranges come back when there are fewer layers than buckets."""
    n = len(sizes)
    if n == 0:
        return []
    if n_buckets < 1:
        raise ValueError("n_buckets must be >= 1")
    cum = np.cumsum(np.asarray(sizes, dtype=np.float64))
    total = cum[-1]
    cuts = [0]
    for k in range(1, min(n_buckets, n)):
        j = int(np.argmin(np.abs(cum - k * total / n_buckets))) + 1
        j = min(max(j, cuts[-1] + 1), n - (min(n_buckets, n) - k))
        cuts.append(j)
    cuts.append(n)
    return [(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]


def bucket_span(layout, bucket: Tuple[int, int]) -> Tuple[int, int]:
    """Element range [a, b) of the flat buffer covered by the layers of ``bucket``."""
    l0, l1 = bucket
    return layout[l0][0], layout[l1 - 1][0] + layout[l1 - 1][1]


def allreduce_bucket(flat, layout, bucket: Tuple[int, int], group=None):
    """Sum over ranks (in place) of one bucket of the flat weight-estimate buffer: one
    collective for all its layers.  The stack calls it on a side stream as soon as the
    bucket's estimates are complete, so the exchange overlaps the remaining layers' work."""
    import torch.distributed as dist
    a, b = bucket_span(layout, bucket)
    dist.all_reduce(flat[a:b], op=dist.ReduceOp.SUM, group=group)
    return flat


def estimate_sharded(x, W, u, cu_local, K: int, sigma: float, gamma: float, seed: int,
                     token_offset: int, layer_id: int = 0, group=None, layer=None):
    """One layer's estimate on this rank's shard (CUDA path), summed over ranks."""
    from . import DustLayer, NoiseKey
    import torch
    N, d_in = x.shape
    d_out = W.shape[0]
    if layer is None:
        layer = DustLayer(N, d_in, d_out, K, x.dtype, x.device)
    cu = torch.as_tensor(cu_local, dtype=torch.int32, device=x.device)
    key = NoiseKey(seed, layer_id, 0, token_offset)
    G_W = layer.estimate(x, W, u, cu, sigma, gamma, key)
    return allreduce_weight_estimate(G_W, group)


def allreduce_probe_scalars(p, group=None):
    """SPSA / MeZO: the sum over ranks of the per-rank projected gradients p [P] (and of the
    perturbed losses, if given the same way).  P scalars per step: the weight-space probes'
    directions are regenerated from the seed on every rank, never sent."""
    import torch.distributed as dist
    dist.all_reduce(p, op=dist.ReduceOp.SUM, group=group)
    return p


def spsa_sharded(x, W, u, P: int, eps: float, seed: int, layer_id: int = 0,
                 probe_offset: int = 0, group=None):
    """The SPSA weight estimate of one layer from this rank's tokens (CUDA path): local probes,
    one all-reduce of P scalars, then the estimate (identical on every rank)."""
    from . import NoiseKey, dust_spsa_estimate, dust_spsa_probe
    key = NoiseKey(seed, layer_id, probe_offset)
    p = dust_spsa_probe(x, W, u, P, eps, key)
    allreduce_probe_scalars(p, group)
    return dust_spsa_estimate(p, P, W.shape[0], W.shape[1], key), p
