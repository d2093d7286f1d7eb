"""Seeded synthetic inputs for the Dust estimator, shared by the CUDA path and the oracle.

This module holds no arithmetic of the estimator itself: it only draws the layer inputs
x, the weights W, the quadratic-readout targets u and the packed sequence boundaries,
and names the five workload shapes.  Both sides read the same stored values.

Recipe (every workload):
  * data generator: numpy PCG64 ``default_rng(1000 + cfg_id)``; draw order x, W, u, then
    segment lengths; for the 48-layer stack the order repeats per layer in the order
    layer_id = 4*block + {0: QKV, 1: O, 2: W_in, 3: W_out}.
  * x ~ N(0, 1), u ~ N(0, 1), W ~ N(0, w_std^2), drawn in float64, rounded to float32 by
    numpy (round to nearest even) and, for bf16 workloads, from float32 to bf16 (round to
    nearest even, the same values as torch's conversion).  The oracle reads the rounded values exactly.
  * noise seed 0x5EED0000 + cfg_id, draw_offset 0, token_offset 0.
  * packed variable-length sequences (the attention-projection workload): lengths are iid
    integers uniform on [256, 2048] drawn until the stream of N tokens is full; the last
    segment is truncated to fit.

The shapes stand in for the transformer layers of the Dust page (koala.ai.kr, "Dust:
역전파 없이 트랜스포머를 사전학습하다", section "설정": GPT-style model, batches of 8 x 2048
tokens); FineWeb and trained weights are not used, only their shapes.
"""
from __future__ import annotations

import dataclasses
import functools
from typing import List, Optional, Sequence

import numpy as np

NOISE_SEED_BASE = 0x5EED0000


@dataclasses.dataclass(frozen=True)
class LayerShape:
    d_in: int
    d_out: int
    layer_id: int
    name: str = ""


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg_id: int
    name: str
    n_seq: int
    seq_len: int
    layers: Sequence[LayerShape]
    K: int
    sigma: float
    gammas: Sequence[float]
    dtype: str                 # "f32" or "bf16"
    w_std: Optional[float]     # None -> 1/sqrt(d_in)
    packed: bool = False       # variable-length packed sequences

    @property
    def N(self) -> int:
        return self.n_seq * self.seq_len

    @property
    def gamma(self) -> float:
        return self.gammas[0]

    @property
    def seed(self) -> int:
        return NOISE_SEED_BASE + self.cfg_id


def _gpt2_stack(n_blocks: int = 12, d: int = 768) -> List[LayerShape]:
    out = []
    for b in range(n_blocks):
        out.append(LayerShape(d, 3 * d, 4 * b + 0, f"block{b}.qkv"))
        out.append(LayerShape(d, d, 4 * b + 1, f"block{b}.o"))
        out.append(LayerShape(d, 4 * d, 4 * b + 2, f"block{b}.w_in"))
        out.append(LayerShape(4 * d, d, 4 * b + 3, f"block{b}.w_out"))
    return out


WORKLOADS = {
    1: Workload(1, "tiny-f32-64x64", 2, 64, [LayerShape(64, 64, 0, "tiny")], 8, 1e-2,
                (0.9, 0.0), "f32", None),
    2: Workload(2, "gpt2s-mlp-win-768x3072", 8, 1024, [LayerShape(768, 3072, 0, "w_in")], 16,
                1e-3, (0.95,), "bf16", 0.02),
    3: Workload(3, "attn-proj-1024x1024-packed", 16, 2048,
                [LayerShape(1024, 1024, 0, "proj")], 32, 1e-3, (0.99,), "bf16", 0.02,
                packed=True),
    4: Workload(4, "large-pop-mlp-2048x8192", 4, 4096, [LayerShape(2048, 8192, 0, "w_in")], 64,
                5e-4, (0.95,), "bf16", 0.02),
    5: Workload(5, "gpt2s-12-block-stack-48-layers", 8, 1024, _gpt2_stack(), 16, 1e-3,
                (0.0, 0.9, 0.99), "bf16", 0.02),
}


def packed_lengths(rng: np.random.Generator, N: int, lo: int = 256, hi: int = 2048) -> np.ndarray:
    """iid integer lengths uniform on [lo, hi] until N tokens are covered; last one truncated."""
    lens = []
    total = 0
    while total < N:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, N - total)
        lens.append(L)
        total += L
    return np.asarray(lens, dtype=np.int64)


def cu_seqlens_from_lengths(lengths: Sequence[int]) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


def to_bf16_bits(a32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even: the top 16 bits after
    adding 0x7fff plus the lowest kept bit (ties go to the even neighbour); a NaN stays a quiet
    NaN.  The same values as torch's float32 -> bfloat16 conversion (checked by a test)."""
    a = np.ascontiguousarray(a32, dtype=np.float32)
    b = a.view(np.uint32)
    out = ((b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))))
           >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = ((b[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _widen(store: np.ndarray, dtype: str) -> np.ndarray:
    """The stored values (float32, or bf16 bit patterns) widened exactly to float64."""
    return store.astype(np.float64) if dtype == "f32" else bf16_bits_to_f64(store)


@dataclasses.dataclass
class LayerData:
    """One layer's inputs. ``*_store`` is what the device receives (float32 array, or bf16
    bit patterns as uint16); ``*_f64`` is the same stored value widened exactly (made on first
    use, so that a large stack that only goes to the device holds no float64 copy)."""
    shape: LayerShape
    dtype: str
    x_store: np.ndarray
    W_store: np.ndarray
    u_store: np.ndarray

    @functools.cached_property
    def x_f64(self) -> np.ndarray:
        return _widen(self.x_store, self.dtype)

    @functools.cached_property
    def W_f64(self) -> np.ndarray:
        return _widen(self.W_store, self.dtype)

    @functools.cached_property
    def u_f64(self) -> np.ndarray:
        return _widen(self.u_store, self.dtype)


def _store(rng, shape, std, dtype):
    a32 = (rng.standard_normal(shape) * std).astype(np.float32)
    return a32 if dtype == "f32" else to_bf16_bits(a32)


def _draw(rng, shape, std, dtype):
    s = _store(rng, shape, std, dtype)
    return s, _widen(s, dtype)


def make_layer(rng: np.random.Generator, shape: LayerShape, N: int, dtype: str,
               w_std: Optional[float]) -> LayerData:
    std_w = (1.0 / np.sqrt(shape.d_in)) if w_std is None else w_std
    xs = _store(rng, (N, shape.d_in), 1.0, dtype)
    Ws = _store(rng, (shape.d_out, shape.d_in), std_w, dtype)
    us = _store(rng, (N, shape.d_out), 1.0, dtype)
    return LayerData(shape, dtype, xs, Ws, us)


@dataclasses.dataclass
class WorkloadData:
    wl: Workload
    layers: List[LayerData]
    cu_seqlens: np.ndarray   # int32 [n_seg + 1]


def generate(cfg_id: int, n_layers: Optional[int] = None) -> WorkloadData:
    """All inputs of workload ``cfg_id`` (``n_layers`` limits the 48-layer stack)."""
    wl = WORKLOADS[cfg_id]
    rng = np.random.default_rng(1000 + cfg_id)
    shapes = list(wl.layers)[: (n_layers or len(wl.layers))]
    layers = [make_layer(rng, s, wl.N, wl.dtype, wl.w_std) for s in shapes]
    if wl.packed:
        cu = cu_seqlens_from_lengths(packed_lengths(rng, wl.N))
    else:
        cu = cu_seqlens_from_lengths([wl.seq_len] * wl.n_seq)
    return WorkloadData(wl, layers, cu)


def custom_layer(seed: int, N: int, d_in: int, d_out: int, dtype: str = "bf16",
                 w_std: Optional[float] = 0.02, layer_id: int = 0) -> LayerData:
    """A seeded layer of arbitrary shape (parity cases with ragged tails)."""
    rng = np.random.default_rng(seed)
    return make_layer(rng, LayerShape(d_in, d_out, layer_id), N, dtype, w_std)


def random_segments(seed: int, N: int, lo: int, hi: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return cu_seqlens_from_lengths(packed_lengths(rng, N, lo, hi))


def dyadic_losses(seed: int, K: int, N: int, scale_bits: int = 8, max_abs: int = 8) -> np.ndarray:
    """float32 [K, N] multiples of 2^-scale_bits with |v| <= max_abs (exact in any sum order
    when the sums stay below 2^24 ulps)."""
    rng = np.random.default_rng(seed)
    m = rng.integers(-max_abs << scale_bits, (max_abs << scale_bits) + 1, size=(K, N))
    return (m.astype(np.float64) / float(1 << scale_bits)).astype(np.float32)


def gaussian_losses(seed: int, K: int, N: int, scale: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((K, N)) * scale).astype(np.float32)


# ------------------------------------------------------------------------------ LM head
@dataclasses.dataclass(frozen=True)
class HeadWorkload:
    """The output layer perturbed on its cached logits: N tokens of hidden width d_model, a
    vocabulary of V entries, noise on the slab [v0, v0 + S), K draws, noise scale sigma,
    discount gamma (0: the head's noise changes only its own token's loss)."""
    name: str
    n_seq: int
    seq_len: int
    d_model: int
    V: int
    v0: int
    S: int
    K: int
    sigma: float
    gamma: float
    dtype: str
    seed: int
    logit_std: float = 2.0

    @property
    def N(self) -> int:
        return self.n_seq * self.seq_len


# The Dust page's setting (section "설정": 4096-entry BPE vocabulary, width 512, batches of
# 8 x 2048 tokens), with a quarter of the vocabulary as the noisy slab and a population of
# 256 draws, larger than the hidden layers' because the head's draws cost no forward pass.
HEAD_WORKLOADS = {
    "head-4096-slab1024": HeadWorkload("head-4096-slab1024", 8, 2048, 512, 4096, 1024, 1024,
                                       256, 1e-2, 0.0, "bf16", NOISE_SEED_BASE + 6),
}


@dataclasses.dataclass
class HeadData:
    wl: HeadWorkload
    z_store: np.ndarray   # logits [N, V] (bf16 bits or float32)
    z_f64: np.ndarray
    y: np.ndarray         # int32 [N] targets, uniform over the vocabulary
    h_store: np.ndarray   # hidden states [N, d_model] (the head's input)
    h_f64: np.ndarray
    cu_seqlens: np.ndarray


def generate_head(wl: HeadWorkload, data_seed: int = 1006) -> HeadData:
    """Logits ~ N(0, logit_std^2), targets uniform on [0, V), hidden states ~ N(0, 1); draw
    order logits, targets, hidden states; sequences of seq_len tokens."""
    rng = np.random.default_rng(data_seed)
    zs, z64 = _draw(rng, (wl.N, wl.V), wl.logit_std, wl.dtype)
    y = rng.integers(0, wl.V, size=wl.N).astype(np.int32)
    hs, h64 = _draw(rng, (wl.N, wl.d_model), 1.0, wl.dtype)
    cu = cu_seqlens_from_lengths([wl.seq_len] * wl.n_seq)
    return HeadData(wl, zs, z64, y, hs, h64, cu)


# ------------------------------------------------------------------------------ attention
@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """A value (or key / gate) projection d_model -> d inside attention, estimated from the
    attention-internal reward: N tokens, K draws, noise scale sigma, discount gamma (close to
    1 for the projections that later tokens read)."""
    name: str
    n_seq: int
    seq_len: int
    d_model: int
    d: int
    K: int
    sigma: float
    gamma: float
    seed: int

    @property
    def N(self) -> int:
        return self.n_seq * self.seq_len


ATTN_WORKLOADS = {
    "attn-v-768": AttnWorkload("attn-v-768", 8, 1024, 768, 768, 16, 1e-3, 0.99,
                               NOISE_SEED_BASE + 7),
}


@dataclasses.dataclass
class AttnData:
    wl: AttnWorkload
    ghat: np.ndarray       # float32 [N, d]: output-error estimate at the attention output
    dO_store: np.ndarray   # bf16 bits [K, N, d]: change of the attention output per draw
    x_store: np.ndarray    # bf16 bits [N, d_model]: the projection's input
    cu_seqlens: np.ndarray


def generate_attn(wl: AttnWorkload, data_seed: int = 1007) -> AttnData:
    """ghat ~ N(0, 1), delta_o ~ N(0, sigma^2) (what the caller's attention recomputation
    would hand over), x ~ N(0, 1); draw order ghat, delta_o, x; sequences of seq_len tokens."""
    rng = np.random.default_rng(data_seed)
    ghat = rng.standard_normal((wl.N, wl.d)).astype(np.float32)
    dO = (rng.standard_normal((wl.K, wl.N, wl.d)) * wl.sigma).astype(np.float32)
    xs, _ = _draw(rng, (wl.N, wl.d_model), 1.0, "bf16")
    return AttnData(wl, ghat, to_bf16_bits(dO), xs,
                    cu_seqlens_from_lengths([wl.seq_len] * wl.n_seq))
