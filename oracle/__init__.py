"""fp64 CPU oracle of the Dust estimator (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product path (``zeroth_order_transformer_b200``) never
imports it and shares no code with it.  The arithmetic lives in ``dust_oracle.c``; this
module only compiles it (gcc, -O2, no fast-math, no FMA contraction) and marshals numpy
arrays through ctypes.

Every function cites the Dust review page (koala.ai.kr, "Dust: 역전파 없이 트랜스포머를
사전학습하다"), section "신용 할당(credit assignment): 보상에서 기울기까지".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dust_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_c_u32p = ctypes.POINTER(ctypes.c_uint32)
_c_f64p = ctypes.POINTER(ctypes.c_double)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle's shared library in place (gcc is part of the image)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_philox4x32_10.argtypes = [_c_u32p, _c_u32p, _c_u32p]
        L.oracle_uniform.argtypes = [ctypes.c_uint32]
        L.oracle_uniform.restype = ctypes.c_double
        L.oracle_philox_batch.argtypes = [_c_u32p, ctypes.c_int64, ctypes.c_uint64, _c_u32p,
                                          _c_f64p]
        L.oracle_normal_stats.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                          ctypes.c_int64, ctypes.c_int32, ctypes.c_double,
                                          ctypes.c_double, _c_f64p, _c_i64p]
        L.oracle_normal_quad.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                         ctypes.c_uint32, ctypes.c_uint32, _c_f64p]
        L.oracle_noisy_linear_loss.argtypes = [
            _c_f64p, _c_f64p, _c_f64p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_double, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
            ctypes.c_uint32, _c_i64p, ctypes.c_int64, _c_f64p, _c_f64p]
        L.oracle_credit.argtypes = [_c_f64p, ctypes.c_int32, ctypes.c_int64, _c_i32p,
                                    ctypes.c_int32, ctypes.c_double, _c_f64p]
        L.oracle_credit_recurrence.argtypes = L.oracle_credit.argtypes
        L.oracle_output_error.argtypes = [
            _c_f64p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
            ctypes.c_double, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32,
            _c_i64p, ctypes.c_int64, _c_i32p, ctypes.c_int32, _c_f64p]
        L.oracle_weight_grad.argtypes = [_c_f64p, _c_f64p, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_int32, _c_f64p]
        L.oracle_sgd_momentum.argtypes = [_c_f64p, _c_f64p, _c_f64p, ctypes.c_int64,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double]
        L.oracle_adam.argtypes = [_c_f64p, _c_f64p, _c_f64p, _c_f64p, ctypes.c_int64,
                                  ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                  ctypes.c_double, ctypes.c_double, ctypes.c_int32]
        L.oracle_noisy_logits_ce.argtypes = [
            _c_f64p, _c_i32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_double, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
            ctypes.c_uint32, _c_i64p, ctypes.c_int64, _c_f64p, _c_f64p]
        L.oracle_attn_reward.argtypes = [_c_f64p, _c_f64p, ctypes.c_int32, ctypes.c_int64,
                                         ctypes.c_int32, _c_f64p]
        L.oracle_discounted_credit.argtypes = L.oracle_credit.argtypes
        L.oracle_spsa_directions.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             _c_f64p]
        L.oracle_spsa_probe.argtypes = [
            _c_f64p, _c_f64p, _c_f64p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_double, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32,
            _c_f64p, _c_f64p, _c_f64p]
        L.oracle_spsa_estimate.argtypes = [_c_f64p, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_uint64,
                                           ctypes.c_uint32, ctypes.c_uint32, _c_f64p]
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_get_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctype)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


# --------------------------------------------------------------------------- noise
def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> np.ndarray:
    """One Philox4x32-10 block (Salmon et al., SC'11): 4 counter words, 2 key words -> 4 words."""
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_p(c, _c_u32p), _p(k, _c_u32p), _p(out, _c_u32p))
    return out


def uniform(w: int) -> float:
    """u(w) = (2 (w >> 9) + 1) 2^-24."""
    return float(lib().oracle_uniform(int(w) & 0xFFFFFFFF))


def philox_batch(ctr: np.ndarray, seed: int, want_normals: bool = True):
    """Words and Box-Muller normals for n counters (array [n, 4] of uint32)."""
    c = np.ascontiguousarray(ctr, dtype=np.uint32).reshape(-1, 4)
    n = c.shape[0]
    words = np.zeros((n, 4), dtype=np.uint32)
    normals = np.zeros((n, 4), dtype=np.float64) if want_normals else None
    lib().oracle_philox_batch(_p(c, _c_u32p), n, int(seed), _p(words, _c_u32p),
                              _p(normals, _c_f64p))
    return words, normals


def normal_stats(seed: int, draw: int, layer: int, n_blocks: int, n_bins: int, lo: float,
                 hi: float):
    """(sum z, sum z^2) and the histogram [n_bins + 2] (under, bins of [lo, hi), over) of the
    4 n_blocks normals of counters (j mod 1024, j / 1024, draw, layer), streamed."""
    sums = np.zeros(2, dtype=np.float64)
    hist = np.zeros(n_bins + 2, dtype=np.int64)
    lib().oracle_normal_stats(int(seed), draw, layer, int(n_blocks), int(n_bins), float(lo),
                              float(hi), _p(sums, _c_f64p), _p(hist, _c_i64p))
    return sums, hist


def noise(seed: int, layer_id: int, N: int, d_out: int, K: int, draw_offset: int = 0,
          token_offset: int = 0) -> np.ndarray:
    """a[i, t, o] for all draws, tokens and channels (small cases only): [K, N, d_out]."""
    nq = (d_out + 3) // 4
    i, t, q = np.meshgrid(np.arange(K, dtype=np.uint32) + np.uint32(draw_offset),
                          np.arange(N, dtype=np.uint32) + np.uint32(token_offset),
                          np.arange(nq, dtype=np.uint32), indexing="ij")
    ctr = np.stack([q, t, i, np.full_like(q, layer_id)], axis=-1).reshape(-1, 4)
    _, z = philox_batch(ctr, seed)
    return z.reshape(K, N, nq * 4)[:, :, :d_out]


# --------------------------------------------------------------------------- estimator
def noisy_linear_loss(x, W, u, K: int, sigma: float, seed: int, layer_id: int = 0,
                      draw_offset: int = 0, token_offset: int = 0, tokens=None):
    """Absolute per-draw losses l[K, n_tok] and clean losses [n_tok] of the quadratic readout
    1/2 ||W x_t + sigma a_t - u_t||^2 (noise equation)."""
    x, W, u = _f64(x), _f64(W), _f64(u)
    N, d_in = x.shape
    d_out = W.shape[0]
    tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n_tok = N if tk is None else tk.shape[0]
    loss = np.zeros((K, n_tok), dtype=np.float64)
    clean = np.zeros(n_tok, dtype=np.float64)
    lib().oracle_noisy_linear_loss(_p(x, _c_f64p), _p(W, _c_f64p), _p(u, _c_f64p), N, d_in,
                                   d_out, K, float(sigma), int(seed), layer_id, draw_offset,
                                   token_offset, _p(tk, _c_i64p), n_tok, _p(loss, _c_f64p),
                                   _p(clean, _c_f64p))
    return loss, clean


def credit(loss, cu_seqlens, gamma: float, route: str = "double_sum") -> np.ndarray:
    """Centred loss then discounted credit r[K, N] (centred-loss and credit equations)."""
    loss = _f64(loss)
    K, N = loss.shape
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    r = np.zeros((K, N), dtype=np.float64)
    fn = lib().oracle_credit if route == "double_sum" else lib().oracle_credit_recurrence
    fn(_p(loss, _c_f64p), K, N, _p(cu, _c_i32p), cu.shape[0] - 1, float(gamma), _p(r, _c_f64p))
    return r


def attn_reward(ghat, dO) -> np.ndarray:
    """c[K, N] = -<ghat_t, dO[i, t]>: the attention-internal reward (Dust page, "간섭 줄이기")."""
    ghat, dO = _f64(ghat), _f64(dO)
    N, d = ghat.shape
    K = dO.shape[0]
    assert dO.shape == (K, N, d)
    c = np.zeros((K, N), dtype=np.float64)
    lib().oracle_attn_reward(_p(ghat, _c_f64p), _p(dO, _c_f64p), K, N, d, _p(c, _c_f64p))
    return c


def discounted_credit(c, cu_seqlens, gamma: float) -> np.ndarray:
    """r[K, N] = sum_{s >= t, same segment} gamma^(s-t) c_s: the credit equation on a given
    reward, without centring."""
    c = _f64(c)
    K, N = c.shape
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    r = np.zeros((K, N), dtype=np.float64)
    lib().oracle_discounted_credit(_p(c, _c_f64p), K, N, _p(cu, _c_i32p), cu.shape[0] - 1,
                                   float(gamma), _p(r, _c_f64p))
    return r


def output_error(r, K_total: int, sigma: float, seed: int, d_out: int, layer_id: int = 0,
                 draw_offset: int = 0, token_offset: int = 0, tokens=None, chans=None):
    """g[n_tok, n_ch] = -(1/(K_total sigma)) sum_i r_t^(i) a_t^(i) (output-error equation)."""
    r = _f64(r)
    K_chunk, N = r.shape
    tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    ch = None if chans is None else np.ascontiguousarray(chans, dtype=np.int32)
    n_tok = N if tk is None else tk.shape[0]
    n_ch = d_out if ch is None else ch.shape[0]
    g = np.zeros((n_tok, n_ch), dtype=np.float64)
    lib().oracle_output_error(_p(r, _c_f64p), K_chunk, K_total, N, d_out, float(sigma),
                              int(seed), layer_id, draw_offset, token_offset, _p(tk, _c_i64p),
                              n_tok, _p(ch, _c_i32p), n_ch, _p(g, _c_f64p))
    return g


def weight_grad(g, x) -> np.ndarray:
    """G_W[d_out, d_in] = sum_t g_t x_t^T, explicit outer-product sum (weight-estimate eq.)."""
    g, x = _f64(g), _f64(x)
    N, d_out = g.shape
    d_in = x.shape[1]
    GW = np.zeros((d_out, d_in), dtype=np.float64)
    lib().oracle_weight_grad(_p(g, _c_f64p), _p(x, _c_f64p), N, d_in, d_out, _p(GW, _c_f64p))
    return GW


def dust_layer(x, W, u, K: int, sigma: float, gamma: float, cu_seqlens, seed: int,
               layer_id: int = 0, token_offset: int = 0):
    """The whole estimator for one layer: returns dict(loss, clean, r, g, G_W)."""
    loss, clean = noisy_linear_loss(x, W, u, K, sigma, seed, layer_id, 0, token_offset)
    r = credit(loss, cu_seqlens, gamma)
    g = output_error(r, K, sigma, seed, W.shape[0], layer_id, 0, token_offset)
    GW = weight_grad(g, x)
    return dict(loss=loss, clean=clean, r=r, g=g, G_W=GW)


# --------------------------------------------------------------------------- optimizers
def sgd_momentum(W, m, G, lr: float, mu: float, wd: float = 0.0):
    """One SGD-with-momentum step (heavy ball): returns new (W, m).  Dust page, "설정"."""
    W, m, G = _f64(W).copy(), _f64(m).copy(), _f64(G)
    lib().oracle_sgd_momentum(_p(W, _c_f64p), _p(m, _c_f64p), _p(G, _c_f64p), W.size, lr, mu, wd)
    return W, m


def adam(W, m, v, G, lr: float, b1: float, b2: float, eps: float, t: int, wd: float = 0.0):
    """One bias-corrected Adam step t >= 1 (Kingma & Ba): returns new (W, m, v)."""
    W, m, v, G = _f64(W).copy(), _f64(m).copy(), _f64(v).copy(), _f64(G)
    lib().oracle_adam(_p(W, _c_f64p), _p(m, _c_f64p), _p(v, _c_f64p), _p(G, _c_f64p), W.size,
                      lr, b1, b2, eps, wd, int(t))
    return W, m, v


# --------------------------------------------------------------------------- LM head
def noisy_logits_ce(z, y, v0: int, S: int, K: int, sigma: float, seed: int, layer_id: int = 0,
                    draw_offset: int = 0, token_offset: int = 0, tokens=None):
    """Absolute cross-entropy losses [K, n_tok] with noise on the logit slab [v0, v0 + S), and the
    clean losses [n_tok] (Dust page, "간섭 줄이기": the LM head perturbed on cached logits)."""
    z = _f64(z)
    N, V = z.shape
    yy = np.ascontiguousarray(y, dtype=np.int32)
    tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    n_tok = N if tk is None else tk.shape[0]
    loss = np.zeros((K, n_tok), dtype=np.float64)
    clean = np.zeros(n_tok, dtype=np.float64)
    lib().oracle_noisy_logits_ce(_p(z, _c_f64p), _p(yy, _c_i32p), N, V, v0, S, K, float(sigma),
                                 int(seed), layer_id, draw_offset, token_offset, _p(tk, _c_i64p),
                                 n_tok, _p(loss, _c_f64p), _p(clean, _c_f64p))
    return loss, clean


# --------------------------------------------------------------------------- SPSA / MeZO
def spsa_directions(seed: int, layer_id: int, P: int, d_out: int, d_in: int,
                    probe_offset: int = 0) -> np.ndarray:
    """The probes' weight-space directions z_j [P, d_out, d_in] (bf16 values, as float64)."""
    Z = np.zeros((P, d_out, d_in), dtype=np.float64)
    lib().oracle_spsa_directions(int(seed), layer_id, probe_offset, P, d_out, d_in,
                                 _p(Z, _c_f64p))
    return Z


def spsa_probe(x, W, u, P: int, eps: float, seed: int, layer_id: int = 0, probe_offset: int = 0):
    """p_j = (L_+ - L_-) / (2 eps) from the two perturbed forwards of each probe; returns
    (p [P], L_+ [P], L_- [P])."""
    x, W, u = _f64(x), _f64(W), _f64(u)
    N, d_in = x.shape
    d_out = W.shape[0]
    p, Lp, Lm = (np.zeros(P, dtype=np.float64) for _ in range(3))
    lib().oracle_spsa_probe(_p(x, _c_f64p), _p(W, _c_f64p), _p(u, _c_f64p), N, d_in, d_out, P,
                            float(eps), int(seed), layer_id, probe_offset, _p(p, _c_f64p),
                            _p(Lp, _c_f64p), _p(Lm, _c_f64p))
    return p, Lp, Lm


def spsa_estimate(p, P_total: int, d_out: int, d_in: int, seed: int, layer_id: int = 0,
                  probe_offset: int = 0) -> np.ndarray:
    """(1/P_total) sum_j p_j z_j [d_out, d_in]."""
    p = _f64(p)
    G = np.zeros((d_out, d_in), dtype=np.float64)
    lib().oracle_spsa_estimate(_p(p, _c_f64p), p.shape[0], P_total, d_out, d_in, int(seed),
                               layer_id, probe_offset, _p(G, _c_f64p))
    return G
