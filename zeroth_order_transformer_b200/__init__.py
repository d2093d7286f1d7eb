"""Python binding of libdust, the B200 implementation of the Dust token-level
node-perturbation gradient estimator for one linear layer.

The binding only marshals arguments: it checks tensors, takes their device pointers and the
current CUDA stream, allocates outputs and workspaces with PyTorch, and calls the C ABI
declared in ``include/dust.h``.  Every step of the estimator runs in the CUDA kernels of
``libdust.so``; there is no other code path.  If the library is missing, every call raises.

Function names follow the C ABI:
  dust_noisy_linear_fwd  per-draw loss change of the noisy layer (noise equation)
  dust_credit            centred loss and discounted credit (centred-loss, credit equations)
  dust_weight_grad       output-error estimate g and weight estimate G_W
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdust.so")

DUST_OK = 0
DUST_ERR_INVALID_ARG = 1
DUST_ERR_UNSUPPORTED = 2
DUST_ERR_CUDA = 3
DUST_ERR_TIMEOUT = 4
DUST_ERR_WORKSPACE = 5

DUST_F32 = 0
DUST_BF16 = 1

DUST_OP_NOISY_LINEAR_FWD = 0
DUST_OP_CREDIT = 1
DUST_OP_WEIGHT_GRAD = 2
DUST_OP_LOGITS_CE = 3
DUST_OP_SPSA_PROBE = 4

EXPORTED_SYMBOLS = (
    "dust_noisy_linear_fwd", "dust_credit", "dust_weight_grad", "dust_workspace_size",
    "dust_status_string", "dust_last_device_error", "dust_debug_philox",
    "dust_debug_credit_skip_publish", "dust_profile_enable", "dust_profile_disable",
    "dust_profile_read", "dust_credit_no_alloc", "dust_noisy_linear_fwd_grouped",
    "dust_credit_grouped", "dust_weight_grad_grouped", "dust_workspace_size_grouped",
    "dust_optimizer_step", "dust_weight_grad_step", "dust_noisy_logits_ce",
    "dust_debug_normal_sum", "dust_debug_fwd_plan", "dust_attn_reward", "dust_discounted_credit",
    "dust_spsa_probe", "dust_spsa_estimate", "dust_noisy_linear_output", "dust_debug_word_sum",
)

DUST_OPT_SGD_MOMENTUM = 1
DUST_OPT_ADAM = 2


class DustError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class dust_noise_key(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("layer_id", ctypes.c_uint32),
                ("draw_offset", ctypes.c_uint32), ("token_offset", ctypes.c_uint32),
                ("channel_offset", ctypes.c_uint32)]


class dust_layer_desc(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("W", ctypes.c_void_p), ("u", ctypes.c_void_p),
                ("d_in", ctypes.c_int32), ("d_out", ctypes.c_int32), ("layer_id", ctypes.c_uint32),
                ("reserved", ctypes.c_uint32), ("dloss", ctypes.c_void_p),
                ("ld_dloss", ctypes.c_int64), ("r", ctypes.c_void_p), ("ld_r", ctypes.c_int64),
                ("G_W", ctypes.c_void_p), ("g_out", ctypes.c_void_p)]


class dust_opt_params(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("step", ctypes.c_int32), ("lr", ctypes.c_float),
                ("momentum", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float)]


def sgd_momentum(lr: float, momentum: float, weight_decay: float = 0.0) -> dust_opt_params:
    return dust_opt_params(DUST_OPT_SGD_MOMENTUM, 0, lr, momentum, 0.0, 0.0, 0.0, weight_decay)


def adam(lr: float, step: int, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
         weight_decay: float = 0.0) -> dust_opt_params:
    return dust_opt_params(DUST_OPT_ADAM, step, lr, 0.0, beta1, beta2, eps, weight_decay)


class NoiseKey(NamedTuple):
    seed: int
    layer_id: int = 0
    draw_offset: int = 0
    token_offset: int = 0
    channel_offset: int = 0

    def c(self) -> dust_noise_key:
        return dust_noise_key(self.seed & 0xFFFFFFFFFFFFFFFF, self.layer_id, self.draw_offset,
                              self.token_offset, self.channel_offset)


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libdust.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdust.so is not built ({LIB_PATH}); run "
                               "`python -m zeroth_order_transformer_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                 ctypes.c_float, ctypes.c_size_t)
        L.dust_noisy_linear_fwd.argtypes = [vp, vp, vp, ctypes.c_int, i64, i32, i32, i32, f32,
                                            dust_noise_key, vp, i64, vp, sz, vp]
        L.dust_credit.argtypes = [vp, i64, i32, i64, vp, i32, f32, vp, i64, vp, sz, vp]
        L.dust_weight_grad.argtypes = [vp, i64, vp, ctypes.c_int, i64, i32, i32, i32, i32, f32,
                                       dust_noise_key, vp, ctypes.c_int, vp, i32, vp, sz, vp]
        L.dust_credit_no_alloc.argtypes = [vp, i64, i32, i64, vp, i32, f32, vp, i64, vp]
        L.dust_credit_no_alloc.restype = ctypes.c_int
        dp = ctypes.POINTER(dust_layer_desc)
        L.dust_noisy_linear_fwd_grouped.argtypes = [dp, i32, i64, i32, f32, dust_noise_key, vp,
                                                    sz, vp]
        L.dust_credit_grouped.argtypes = [dp, i32, i32, i64, vp, i32, f32, vp, sz, vp]
        L.dust_weight_grad_grouped.argtypes = [dp, i32, i64, i32, i32, f32, dust_noise_key,
                                               ctypes.c_int, i32, vp, sz, vp]
        L.dust_workspace_size_grouped.argtypes = [ctypes.c_int, dp, i32, i64, i32]
        L.dust_workspace_size_grouped.restype = sz
        for name in ("dust_noisy_linear_fwd_grouped", "dust_credit_grouped",
                     "dust_weight_grad_grouped"):
            getattr(L, name).restype = ctypes.c_int
        op = ctypes.POINTER(dust_opt_params)
        L.dust_optimizer_step.argtypes = [op, vp, vp, vp, vp, vp, i64, vp]
        L.dust_optimizer_step.restype = ctypes.c_int
        L.dust_weight_grad_step.argtypes = [vp, i64, vp, ctypes.c_int, i64, i32, i32, i32, i32,
                                            f32, dust_noise_key, vp, ctypes.c_int, vp, i32, op, vp,
                                            vp, vp, vp, vp, sz, vp]
        L.dust_weight_grad_step.restype = ctypes.c_int
        L.dust_noisy_logits_ce.argtypes = [vp, i64, ctypes.c_int, vp, i64, i32, i32, i32, i32,
                                           f32, dust_noise_key, vp, i64, vp, sz, vp]
        L.dust_noisy_logits_ce.restype = ctypes.c_int
        L.dust_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int, i64, i32, i32, i32]
        L.dust_workspace_size.restype = sz
        L.dust_status_string.argtypes = [ctypes.c_int]
        L.dust_status_string.restype = ctypes.c_char_p
        L.dust_last_device_error.argtypes = [vp, ctypes.POINTER(i32)]
        L.dust_debug_philox.argtypes = [vp, i64, ctypes.c_uint64, vp, vp, vp]
        L.dust_attn_reward.argtypes = [vp, i64, vp, i64, ctypes.c_int, i64, i32, i32, vp, i64,
                                       vp]
        L.dust_attn_reward.restype = ctypes.c_int
        L.dust_discounted_credit.argtypes = [vp, i64, i32, i64, vp, i32, f32, vp, i64, vp, sz,
                                             vp]
        L.dust_discounted_credit.restype = ctypes.c_int
        L.dust_noisy_linear_output.argtypes = [vp, vp, ctypes.c_int, i64, i32, i32, i32, f32,
                                               dust_noise_key, vp, ctypes.c_int, i64, vp]
        L.dust_noisy_linear_output.restype = ctypes.c_int
        L.dust_spsa_probe.argtypes = [vp, vp, vp, ctypes.c_int, i64, i32, i32, i32, f32,
                                      dust_noise_key, vp, vp, vp, vp, sz, vp]
        L.dust_spsa_probe.restype = ctypes.c_int
        L.dust_spsa_estimate.argtypes = [vp, i32, i32, i32, i32, dust_noise_key, vp, ctypes.c_int,
                                         vp]
        L.dust_spsa_estimate.restype = ctypes.c_int
        L.dust_debug_normal_sum.argtypes = [dust_noise_key, i64, i32, vp, vp]
        L.dust_debug_normal_sum.restype = ctypes.c_int
        L.dust_debug_word_sum.argtypes = [dust_noise_key, i64, i32, vp, vp]
        L.dust_debug_word_sum.restype = ctypes.c_int
        L.dust_debug_credit_skip_publish.argtypes = [i32]
        L.dust_debug_credit_skip_publish.restype = None
        L.dust_debug_fwd_plan.argtypes = [i64, i32, i32, vp, i32, ctypes.POINTER(i32),
                                          ctypes.POINTER(i32)]
        L.dust_debug_fwd_plan.restype = ctypes.c_int
        L.dust_profile_enable.argtypes = [i32]
        L.dust_profile_enable.restype = ctypes.c_int
        L.dust_profile_disable.argtypes = []
        L.dust_profile_disable.restype = None
        L.dust_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p),
                                        ctypes.POINTER(ctypes.c_float), i32]
        L.dust_profile_read.restype = i32
        for name in ("dust_noisy_linear_fwd", "dust_credit", "dust_weight_grad",
                     "dust_last_device_error", "dust_debug_philox"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().dust_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != DUST_OK:
        raise DustError(status, where)


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return DUST_BF16
    if t.dtype == torch.float32:
        return DUST_F32
    raise TypeError(f"unsupported dtype {t.dtype}; layers are bf16 or fp32")


def _cuda(t, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _cuda_rows(t, name: str):
    """A CUDA matrix whose rows are contiguous; rows may be further apart (the row stride is
    passed as the leading dimension)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a matrix with contiguous rows")
    return t


def _stream(device, stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def _workspace(ws, nbytes: int, device):
    torch = _torch()
    if nbytes == 0:
        return None, 0
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws, ws.numel() * ws.element_size()


def dust_workspace_size(op: int, dtype: int, N: int, d_in: int, d_out: int, K: int) -> int:
    return int(lib().dust_workspace_size(op, dtype, N, d_in, d_out, K))


def dust_noisy_linear_fwd(x, W, u, K: int, sigma: float, key: NoiseKey, dloss=None,
                          workspace=None, stream=None):
    """Per-draw loss change dloss[K, N] (fp32) of the layer W x_t + sigma a_t against u_t."""
    torch = _torch()
    _cuda(x, "x"), _cuda(W, "W"), _cuda(u, "u")
    N, d_in = x.shape
    d_out = W.shape[0]
    if W.shape != (d_out, d_in) or u.shape != (N, d_out) or not (x.dtype == W.dtype == u.dtype):
        raise ValueError("shapes/dtypes: x [N, d_in], W [d_out, d_in], u [N, d_out], one dtype")
    dt = _dtype_code(x)
    if dloss is None:
        dloss = torch.empty((K, N), dtype=torch.float32, device=x.device)
    _cuda_rows(dloss, "dloss")
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_NOISY_LINEAR_FWD, dt, N, d_in,
                                                       d_out, K), x.device)
    st = lib().dust_noisy_linear_fwd(x.data_ptr(), W.data_ptr(), u.data_ptr(), dt, N, d_in,
                                     d_out, K, float(sigma), key.c(), dloss.data_ptr(),
                                     dloss.stride(0), ws.data_ptr() if ws is not None else None,
                                     nb, _stream(x.device, stream))
    _check(st, "dust_noisy_linear_fwd")
    return dloss


def dust_noisy_logits_ce(z, y, v0: int, S: int, K: int, sigma: float, key: NoiseKey,
                         dloss=None, workspace=None, stream=None):
    """Per-draw change of the full-vocabulary cross-entropy dloss[K, N] when noise is added to
    the cached logits of the slab [v0, v0 + S) (LM-head perturbation)."""
    torch = _torch()
    _cuda(z, "z"), _cuda(y, "y")
    if y.dtype != torch.int32:
        raise TypeError("y must be int32")
    N, V = z.shape
    dt = _dtype_code(z)
    if dloss is None:
        dloss = torch.empty((K, N), dtype=torch.float32, device=z.device)
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_LOGITS_CE, dt, N, V, S, K),
                        z.device)
    st = lib().dust_noisy_logits_ce(z.data_ptr(), z.stride(0), dt, y.data_ptr(), N, V, v0, S, K,
                                    float(sigma), key.c(), dloss.data_ptr(), dloss.stride(0),
                                    ws.data_ptr() if ws is not None else None, nb,
                                    _stream(z.device, stream))
    _check(st, "dust_noisy_logits_ce")
    return dloss


def dust_credit(loss, cu_seqlens, gamma: float, r=None, workspace=None, stream=None):
    """Credit r[K, N] from losses [K, N] and int32 cu_seqlens [n_seq + 1] (device)."""
    torch = _torch()
    _cuda_rows(loss, "loss"), _cuda(cu_seqlens, "cu_seqlens")
    if loss.dtype != torch.float32 or cu_seqlens.dtype != torch.int32:
        raise TypeError("loss must be float32 and cu_seqlens int32")
    K, N = loss.shape
    if r is None:
        r = torch.empty((K, N), dtype=torch.float32, device=loss.device)
    _cuda_rows(r, "r")
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_CREDIT, DUST_F32, N, 0, 0, K),
                        loss.device)
    st = lib().dust_credit(loss.data_ptr(), loss.stride(0), K, N, cu_seqlens.data_ptr(),
                           cu_seqlens.numel() - 1, float(gamma), r.data_ptr(), r.stride(0),
                           ws.data_ptr() if ws is not None else None, nb,
                           _stream(loss.device, stream))
    _check(st, "dust_credit")
    return r


def dust_attn_reward(ghat, delta_o, c=None, stream=None):
    """Attention-internal reward c[K, N] = -<ghat_t, delta_o[i, t]> from the fp32 output-error
    estimate ghat [N, d] at the attention output and delta_o [K, N, d] (bf16 or fp32)."""
    torch = _torch()
    _cuda(ghat, "ghat")
    if not delta_o.is_cuda:
        raise ValueError("delta_o must be a CUDA tensor")
    if ghat.dtype != torch.float32:
        raise TypeError("ghat must be float32")
    K, N, d = delta_o.shape
    if tuple(ghat.shape) != (N, d) or delta_o.stride(2) != 1 or delta_o.stride(0) != N * delta_o.stride(1):
        raise ValueError("ghat must be [N, d] and delta_o [K, N, d] with rows N * ld apart")
    if c is None:
        c = torch.empty((K, N), dtype=torch.float32, device=ghat.device)
    st = lib().dust_attn_reward(ghat.data_ptr(), ghat.stride(0), delta_o.data_ptr(),
                                delta_o.stride(1), _dtype_code(delta_o), N, d, K, c.data_ptr(),
                                c.stride(0), _stream(ghat.device, stream))
    _check(st, "dust_attn_reward")
    return c


def dust_discounted_credit(c, cu_seqlens, gamma: float, r=None, workspace=None, stream=None):
    """The credit equation on a given reward c [K, N] (no centring): r[K, N]."""
    torch = _torch()
    _cuda(c, "c"), _cuda(cu_seqlens, "cu_seqlens")
    if c.dtype != torch.float32 or cu_seqlens.dtype != torch.int32:
        raise TypeError("c must be float32 and cu_seqlens int32")
    K, N = c.shape
    if r is None:
        r = torch.empty((K, N), dtype=torch.float32, device=c.device)
    _cuda(r, "r")
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_CREDIT, DUST_F32, N, 0, 0, K),
                        c.device)
    st = lib().dust_discounted_credit(c.data_ptr(), c.stride(0), K, N, cu_seqlens.data_ptr(),
                                      cu_seqlens.numel() - 1, float(gamma), r.data_ptr(),
                                      r.stride(0), ws.data_ptr() if ws is not None else None,
                                      nb, _stream(c.device, stream))
    _check(st, "dust_discounted_credit")
    return r


def dust_noisy_linear_output(x, W, K: int, sigma: float, key: NoiseKey, y_out=None,
                             out_dtype=None, stream=None):
    """The perturbed outputs y_out[K, N, d_out] = W x_t + sigma a_t^(i) (fp32 by default, or
    out_dtype=torch.bfloat16), with the noise of dust_noisy_linear_fwd for the same key."""
    torch = _torch()
    _cuda(x, "x"), _cuda(W, "W")
    N, d_in = x.shape
    d_out = W.shape[0]
    if y_out is None:
        y_out = torch.empty((K, N, d_out), dtype=out_dtype or torch.float32, device=x.device)
    _cuda(y_out, "y_out")
    st = lib().dust_noisy_linear_output(x.data_ptr(), W.data_ptr(), _dtype_code(x), N, d_in,
                                        d_out, K, float(sigma), key.c(), y_out.data_ptr(),
                                        _dtype_code(y_out), y_out.stride(1),
                                        _stream(x.device, stream))
    _check(st, "dust_noisy_linear_output")
    return y_out


def dust_spsa_probe(x, W, u, P: int, eps: float, key: NoiseKey, p=None, losses: bool = False,
                    workspace=None, stream=None):
    """SPSA / MeZO probe: p[P] = (L_+ - L_-) / (2 eps) for the weight directions z_j of
    draws key.draw_offset .. + P; with losses=True also returns L_+ and L_- [P]."""
    torch = _torch()
    _cuda(x, "x"), _cuda(W, "W"), _cuda(u, "u")
    N, d_in = x.shape
    d_out = W.shape[0]
    dt = _dtype_code(x)
    if p is None:
        p = torch.empty(P, dtype=torch.float32, device=x.device)
    Lp = torch.empty(P, dtype=torch.float32, device=x.device) if losses else None
    Lm = torch.empty(P, dtype=torch.float32, device=x.device) if losses else None
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_SPSA_PROBE, dt, N, d_in, d_out, P),
                        x.device)
    st = lib().dust_spsa_probe(x.data_ptr(), W.data_ptr(), u.data_ptr(), dt, N, d_in, d_out, P,
                               float(eps), key.c(), p.data_ptr(), _ptr(Lp), _ptr(Lm),
                               ws.data_ptr() if ws is not None else None, nb,
                               _stream(x.device, stream))
    _check(st, "dust_spsa_probe")
    return (p, Lp, Lm) if losses else p


def dust_spsa_estimate(p, P_total: int, d_out: int, d_in: int, key: NoiseKey, G=None,
                       accumulate: bool = False, stream=None):
    """G [d_out, d_in] (+)= (1/P_total) sum_j p[j] z_j."""
    torch = _torch()
    _cuda(p, "p")
    if G is None:
        G = torch.empty((d_out, d_in), dtype=torch.float32, device=p.device)
        accumulate = False
    _cuda(G, "G")
    st = lib().dust_spsa_estimate(p.data_ptr(), p.numel(), P_total, d_in, d_out, key.c(),
                                  G.data_ptr(), 1 if accumulate else 0, _stream(p.device, stream))
    _check(st, "dust_spsa_estimate")
    return G


def dust_credit_no_alloc(loss, cu_seqlens, gamma: float, r, stream=None):
    """dust_credit with the library's static 4 MiB scratch instead of a workspace, for callers
    that cannot allocate device memory; ``r`` must be given (float32 [K, N], rows contiguous,
    rows may be further apart, as may those of ``loss``).  Calls that overlap on the GPU share
    the scratch and race: serialize them."""
    torch = _torch()
    _cuda_rows(loss, "loss"), _cuda(cu_seqlens, "cu_seqlens"), _cuda_rows(r, "r")
    if loss.dtype != torch.float32 or r.dtype != torch.float32 or cu_seqlens.dtype != torch.int32:
        raise TypeError("loss and r must be float32 and cu_seqlens int32")
    K, N = loss.shape
    if tuple(r.shape) != (K, N):
        raise ValueError(f"r must be [K, N] = [{K}, {N}] like loss, got {tuple(r.shape)}")
    st = lib().dust_credit_no_alloc(loss.data_ptr(), loss.stride(0), K, N, cu_seqlens.data_ptr(),
                                    cu_seqlens.numel() - 1, float(gamma), r.data_ptr(),
                                    r.stride(0), _stream(loss.device, stream))
    _check(st, "dust_credit_no_alloc")
    return r


G_TERMS = 2  # default: g enters the bf16 contraction as hi + lo terms


def dust_weight_grad(r, x, d_out: int, K_total: int, sigma: float, key: NoiseKey, G_W=None,
                     accumulate: bool = False, g_out=None, workspace=None, stream=None,
                     g_terms: int = G_TERMS) -> Tuple[object, Optional[object]]:
    """G_W[d_out, d_in] (fp32) and, if g_out is a tensor or True, g[N, d_out] (fp32).  For bf16
    x, g enters the tensor cores as ``g_terms`` bf16 terms (2: hi + lo; 1: rounded once)."""
    torch = _torch()
    _cuda_rows(r, "r"), _cuda(x, "x")
    K_chunk, N = r.shape
    d_in = x.shape[1]
    dt = _dtype_code(x)
    if G_W is None:
        G_W = torch.empty((d_out, d_in), dtype=torch.float32, device=x.device)
        accumulate = False
    _cuda(G_W, "G_W")
    if g_out is True:
        g_out = torch.empty((N, d_out), dtype=torch.float32, device=x.device)
    if g_out is False:
        g_out = None
    need = dust_workspace_size(DUST_OP_WEIGHT_GRAD, dt, N, d_in, d_out, K_chunk)
    if dt == DUST_F32 and g_out is not None:
        need = 0
    ws, nb = _workspace(workspace, need, x.device)
    st = lib().dust_weight_grad(r.data_ptr(), r.stride(0), x.data_ptr(), dt, N, d_in, d_out,
                                K_chunk, K_total, float(sigma), key.c(), G_W.data_ptr(),
                                1 if accumulate else 0,
                                g_out.data_ptr() if g_out is not None else None, int(g_terms),
                                ws.data_ptr() if ws is not None else None, nb,
                                _stream(x.device, stream))
    _check(st, "dust_weight_grad")
    return G_W, g_out


def _ptr(t):
    return t.data_ptr() if t is not None else None


def dust_optimizer_step(opt: dust_opt_params, G, W, m, v=None, W_bf16=None, stream=None):
    """One optimizer step in place on fp32 W, m (and v for Adam) from the estimate G."""
    for t, nm in ((G, "G"), (W, "W"), (m, "m")):
        _cuda(t, nm)
    st = lib().dust_optimizer_step(ctypes.byref(opt), G.data_ptr(), W.data_ptr(), _ptr(W_bf16),
                                   m.data_ptr(), _ptr(v), W.numel(), _stream(W.device, stream))
    _check(st, "dust_optimizer_step")
    return W


def dust_weight_grad_step(r, x, d_out: int, K_total: int, sigma: float, key: NoiseKey,
                          opt: dust_opt_params, W, m, v=None, W_bf16=None, G_W=None,
                          accumulate: bool = False, g_out=None, workspace=None, stream=None,
                          g_terms: int = G_TERMS):
    """dust_weight_grad with the optimizer step fused into the pass that finishes G_W."""
    _cuda(r, "r"), _cuda(x, "x"), _cuda(W, "W"), _cuda(m, "m")
    K_chunk, N = r.shape
    d_in = x.shape[1]
    dt = _dtype_code(x)
    ws, nb = _workspace(workspace, dust_workspace_size(DUST_OP_WEIGHT_GRAD, dt, N, d_in, d_out,
                                                       K_chunk), x.device)
    st = lib().dust_weight_grad_step(r.data_ptr(), r.stride(0), x.data_ptr(), dt, N, d_in, d_out,
                                     K_chunk, K_total, float(sigma), key.c(), _ptr(G_W),
                                     1 if accumulate else 0, _ptr(g_out), int(g_terms),
                                     ctypes.byref(opt),
                                     W.data_ptr(), _ptr(W_bf16), m.data_ptr(), _ptr(v),
                                     ws.data_ptr() if ws is not None else None, nb,
                                     _stream(x.device, stream))
    _check(st, "dust_weight_grad_step")
    return W


def dust_last_device_error(stream=None, device=None) -> Tuple[int, int]:
    """(status, info) of the device error word, which is then cleared."""
    torch = _torch()
    dev = device if device is not None else torch.cuda.current_device()
    info = ctypes.c_int32(0)
    st = lib().dust_last_device_error(_stream(dev, stream), ctypes.byref(info))
    return int(st), int(info.value)


def dust_debug_philox(ctr, seed: int, stream=None):
    """Words (uint32 as int64) and fp32 normals for counters ctr [n, 4] (uint32 as int32)."""
    torch = _torch()
    _cuda(ctr, "ctr")
    n = ctr.shape[0]
    words = torch.empty((n, 4), dtype=torch.int32, device=ctr.device)
    normals = torch.empty((n, 4), dtype=torch.float32, device=ctr.device)
    st = lib().dust_debug_philox(ctr.data_ptr(), n, seed & 0xFFFFFFFFFFFFFFFF, words.data_ptr(),
                                 normals.data_ptr(), _stream(ctr.device, stream))
    _check(st, "dust_debug_philox")
    return words, normals


def dust_debug_normal_sum(key: NoiseKey, n: int, n_quads: int, out=None, device=None,
                          stream=None):
    """out[g] = sum of the 4 n_quads normals of token key.token_offset + g (draw
    key.draw_offset, channels from key.channel_offset): the generator-only throughput probe."""
    torch = _torch()
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=device or "cuda")
    _cuda(out, "out")
    st = lib().dust_debug_normal_sum(key.c(), n, n_quads, out.data_ptr(),
                                     _stream(out.device, stream))
    _check(st, "dust_debug_normal_sum")
    return out


def dust_debug_word_sum(key: NoiseKey, n: int, n_blocks: int, out=None, device=None,
                        stream=None):
    """out[g] (int32 bits of uint32) = XOR of the words of the Philox blocks (channel quad
    key.channel_offset / 4 + j, token key.token_offset + g, draw key.draw_offset), j < n_blocks:
    the generator's integer part alone, as a throughput probe."""
    torch = _torch()
    if out is None:
        out = torch.empty(n, dtype=torch.int32, device=device or "cuda")
    _cuda(out, "out")
    st = lib().dust_debug_word_sum(key.c(), n, n_blocks, out.data_ptr(),
                                   _stream(out.device, stream))
    _check(st, "dust_debug_word_sum")
    return out


def dust_debug_fwd_plan(N: int, K: int, d_outs, sms: int):
    """(persistent, tail split) of the bf16 forward for layers of output widths `d_outs` on a
    device with `sms` SMs (host only; no device needed)."""
    arr = (ctypes.c_int32 * len(d_outs))(*[int(d) for d in d_outs])
    p, sp = ctypes.c_int32(0), ctypes.c_int32(0)
    st = lib().dust_debug_fwd_plan(int(N), int(K), len(d_outs), ctypes.cast(arr, ctypes.c_void_p),
                                   int(sms), ctypes.byref(p), ctypes.byref(sp))
    _check(st, "dust_debug_fwd_plan")
    return bool(p.value), sp.value


def dust_debug_credit_skip_publish(block: int) -> None:
    lib().dust_debug_credit_skip_publish(int(block))


def dust_profile_enable(capacity: int) -> None:
    _check(lib().dust_profile_enable(int(capacity)), "dust_profile_enable")


def dust_profile_disable() -> None:
    lib().dust_profile_disable()


def dust_profile_read(max_records: int = 1 << 16):
    """[(kernel name, milliseconds)] of the launches recorded since enabling (synchronizes)."""
    names = (ctypes.c_char_p * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = lib().dust_profile_read(names, ms, max_records)
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def _sequence_cuts(cu, N: int, chunks: int):
    """Token cuts [0, ..., N] at sequence ends near k N / chunks, kept at multiples of 4 tokens
    so that every run's row and column views stay 16-byte aligned."""
    import numpy as np
    ends = cu[(cu % 4 == 0) & (cu > 0) & (cu < N)]
    cuts = [0]
    for c in range(1, chunks):
        if ends.size == 0:
            break
        e = int(ends[int(np.argmin(np.abs(ends - N * c / chunks)))])
        if e > cuts[-1]:
            cuts.append(e)
    cuts.append(N)
    return cuts


class DustStack:
    """Many bf16 layers sharing one token batch (a transformer block stack), estimated with the
    grouped calls: one launch per step for up to 64 layers.  ``layers`` is a list of
    (x, W, u, layer_id) device tensors; outputs live in ``dloss[l]``, ``r[l]``, ``G_W[l]``.
    The weight estimates are views of one flat fp32 buffer ``G_W_flat`` (layer l at
    ``layout[l]``), so that consecutive layers can be exchanged between ranks in one call."""

    def __init__(self, layers, K: int, want_g: bool = False, g_terms: int = G_TERMS):
        from . import distributed
        torch = _torch()
        self.K = K
        self.g_terms = g_terms
        self.layers = layers
        x0 = layers[0][0]
        self.N = x0.shape[0]
        dev = x0.device
        n = len(layers)
        self.dloss = [torch.empty((K, self.N), dtype=torch.float32, device=dev) for _ in range(n)]
        self.r = [torch.empty((K, self.N), dtype=torch.float32, device=dev) for _ in range(n)]
        self.layout, total = distributed.flat_layout([(W.shape[0], W.shape[1])
                                                      for (_, W, _, _) in layers])
        self.G_W_flat = torch.empty(total, dtype=torch.float32, device=dev)
        self.G_W = [self.G_W_flat[o:o + m].view(W.shape[0], W.shape[1])
                    for (o, m), (_, W, _, _) in zip(self.layout, layers)]
        self.g = ([torch.empty((self.N, W.shape[0]), dtype=torch.float32, device=dev)
                   for (_, W, _, _) in layers] if want_g else None)
        self.desc = (dust_layer_desc * n)()
        for l, (x, W, u, layer_id) in enumerate(layers):
            for t, nm in ((x, "x"), (W, "W"), (u, "u")):
                _cuda(t, nm)
                if t.dtype != torch.bfloat16:
                    raise TypeError("grouped calls take bf16 layers")
            if x.shape[0] != self.N or u.shape != (self.N, W.shape[0]) or x.shape[1] != W.shape[1]:
                raise ValueError("layer shapes: x [N, d_in], W [d_out, d_in], u [N, d_out]")
            d = self.desc[l]
            d.x, d.W, d.u = x.data_ptr(), W.data_ptr(), u.data_ptr()
            d.d_in, d.d_out = x.shape[1], W.shape[0]
            d.layer_id, d.reserved = layer_id, 0
            d.dloss, d.ld_dloss = self.dloss[l].data_ptr(), self.N
            d.r, d.ld_r = self.r[l].data_ptr(), self.N
            d.G_W = self.G_W[l].data_ptr()
            d.g_out = self.g[l].data_ptr() if want_g else None
        self.ws = torch.empty(max(self._ws_need(self.desc, n, self.N), 256), dtype=torch.uint8,
                              device=dev)
        self._comm = None

    def _ws_need(self, desc, n: int, N: int) -> int:
        return max(int(lib().dust_workspace_size_grouped(op, desc, n, N, self.K))
                   for op in range(3))

    @staticmethod
    def _sub(desc, l0: int):
        """Pointer to descriptor l0 of a descriptor array (a bucket of consecutive layers)."""
        return ctypes.cast(ctypes.addressof(desc) + l0 * ctypes.sizeof(dust_layer_desc),
                           ctypes.POINTER(dust_layer_desc))

    def _weight_grad(self, desc, N: int, key, accumulate: bool, s: int, reduce, buckets: int):
        """The grouped weight estimate; with ``reduce``, in buckets of consecutive layers, each
        bucket's span of G_W_flat handed to ``reduce`` on a side stream as soon as its launch
        is queued, so the exchange overlaps the later buckets' work."""
        from . import distributed
        torch = _torch()
        n = len(self.layers)
        nb = self.ws.numel()
        if reduce is None:
            _check(lib().dust_weight_grad_grouped(desc, n, N, self.K, self.K, float(self.sigma),
                                                  key, 1 if accumulate else 0, self.g_terms,
                                                  self.ws.data_ptr(), nb, s),
                   "dust_weight_grad_grouped")
            return
        dev = self.ws.device
        comp = torch.cuda.current_stream(dev)
        if self._comm is None:
            self._comm = torch.cuda.Stream(device=dev)
        plan = distributed.plan_buckets([m for _, m in self.layout], buckets)
        for l0, l1 in plan:
            sub = self._sub(desc, l0)
            need = int(lib().dust_workspace_size_grouped(DUST_OP_WEIGHT_GRAD, sub, l1 - l0, N,
                                                         self.K))
            if need > nb:
                raise RuntimeError("stack workspace too small for a bucket")
            _check(lib().dust_weight_grad_grouped(sub, l1 - l0, N, self.K, self.K,
                                                  float(self.sigma), key,
                                                  1 if accumulate else 0, self.g_terms,
                                                  self.ws.data_ptr(), nb, s),
                   "dust_weight_grad_grouped")
            ev = torch.cuda.Event()
            ev.record(comp)
            self._comm.wait_event(ev)
            with torch.cuda.stream(self._comm):
                a, b = distributed.bucket_span(self.layout, (l0, l1))
                reduce(self.G_W_flat[a:b])
        comp.wait_stream(self._comm)

    def estimate(self, cu_seqlens, sigma: float, gamma: float, seed: int, draw_offset: int = 0,
                 token_offset: int = 0, stream=None, reduce=None, buckets: int = 12):
        """Forward, credit and weight estimate of every layer on the device inputs.  ``reduce``
        (optional, e.g. a sum over data-parallel ranks) is applied to G_W_flat in ``buckets``
        spans of consecutive layers, overlapped with the remaining weight estimates; it must
        run on the current stream (torch collectives do).  ``stream`` must be None (the
        current stream) when ``reduce`` is given."""
        if reduce is not None and stream is not None:
            raise ValueError("reduce runs against the current stream; pass stream=None")
        n = len(self.layers)
        s = _stream(self.ws.device, stream)
        nb = self.ws.numel()
        self.sigma = sigma
        key = NoiseKey(seed, 0, draw_offset, token_offset).c()
        _check(lib().dust_noisy_linear_fwd_grouped(self.desc, n, self.N, self.K, float(sigma), key,
                                                   self.ws.data_ptr(), nb, s),
               "dust_noisy_linear_fwd_grouped")
        _check(lib().dust_credit_grouped(self.desc, n, self.K, self.N, cu_seqlens.data_ptr(),
                                         cu_seqlens.numel() - 1, float(gamma), self.ws.data_ptr(),
                                         nb, s), "dust_credit_grouped")
        self._weight_grad(self.desc, self.N, key, False, s, reduce, buckets)
        return self.G_W

    def estimate_from_host(self, host_layers, cu_seqlens, sigma: float, gamma: float,
                           seed: int, G_host=None, chunks: int = 12, reduce=None,
                           draw_offset: int = 0, token_offset: int = 0):
        """The estimate from inputs in pinned host memory (``host_layers``: one (x, W, u) per
        layer, the shapes of the stack's device tensors, which receive them), pipelined over
        ``chunks`` buckets of consecutive layers of about equal input bytes: a copy stream
        uploads bucket after bucket; each bucket goes through the grouped forward, credit and
        weight estimate as soon as its inputs are in; its span of G_W_flat is copied back on a
        third stream (into ``G_host``, pinned, allocated if None) while the later buckets are
        uploaded and estimated.  ``reduce`` (optional, e.g. the sum over data-parallel ranks)
        is applied to each bucket's span on a side stream before it is copied back.
        Synchronises."""
        from . import distributed
        import numpy as np
        torch = _torch()
        dev = self.ws.device
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        N = int(cu[-1])
        if N != self.N or len(host_layers) != len(self.layers):
            raise ValueError("host inputs do not match the stack")
        self.sigma = sigma
        if not hasattr(self, "_copy"):
            self._copy = torch.cuda.Stream(device=dev)
            self._back = torch.cuda.Stream(device=dev)
        comp = torch.cuda.current_stream(dev)
        cu_d = torch.from_numpy(cu.astype(np.int32)).pin_memory().to(dev, non_blocking=True)
        sizes = [sum(t.numel() * t.element_size() for t in h) for h in host_layers]
        plan = distributed.plan_buckets(sizes, chunks)
        ready = []
        self._copy.wait_stream(comp)  # the uploads start after the work already queued
        with torch.cuda.stream(self._copy):
            for l0, l1 in plan:
                for (x, W, u, _), (hx, hW, hu) in zip(self.layers[l0:l1], host_layers[l0:l1]):
                    W.copy_(hW, non_blocking=True)
                    x.copy_(hx, non_blocking=True)
                    u.copy_(hu, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self._copy)
                ready.append(ev)
        if G_host is None:
            G_host = torch.empty(self.G_W_flat.shape, dtype=torch.float32, pin_memory=True)
        nb = self.ws.numel()
        s = _stream(dev, None)
        key = NoiseKey(seed, 0, draw_offset, token_offset).c()
        if reduce is not None and self._comm is None:
            self._comm = torch.cuda.Stream(device=dev)
        for (l0, l1), ev in zip(plan, ready):
            comp.wait_event(ev)
            n = l1 - l0
            sub = self._sub(self.desc, l0)
            if self._ws_need(sub, n, N) > nb:
                raise RuntimeError("stack workspace too small for a bucket")
            _check(lib().dust_noisy_linear_fwd_grouped(sub, n, N, self.K, float(sigma), key,
                                                       self.ws.data_ptr(), nb, s),
                   "dust_noisy_linear_fwd_grouped")
            _check(lib().dust_credit_grouped(sub, n, self.K, N, cu_d.data_ptr(), cu_d.numel() - 1,
                                             float(gamma), self.ws.data_ptr(), nb, s),
                   "dust_credit_grouped")
            _check(lib().dust_weight_grad_grouped(sub, n, N, self.K, self.K, float(sigma), key, 0,
                                                  self.g_terms, self.ws.data_ptr(), nb, s),
                   "dust_weight_grad_grouped")
            a, b = distributed.bucket_span(self.layout, (l0, l1))
            done = torch.cuda.Event()
            done.record(comp)
            src = comp
            if reduce is not None:
                self._comm.wait_event(done)
                with torch.cuda.stream(self._comm):
                    reduce(self.G_W_flat[a:b])
                src = self._comm
            self._back.wait_stream(src)
            with torch.cuda.stream(self._back):
                G_host[a:b].copy_(self.G_W_flat[a:b], non_blocking=True)
        comp.wait_stream(self._back)
        comp.synchronize()
        return G_host


class DustLayer:
    """One layer's estimator with workspaces kept between calls (fwd -> credit -> weight grad)."""

    def __init__(self, N: int, d_in: int, d_out: int, K: int, dtype, device):
        torch = _torch()
        dt = DUST_BF16 if dtype == torch.bfloat16 else DUST_F32
        self.N, self.d_in, self.d_out, self.K = N, d_in, d_out, K
        nbytes = max(dust_workspace_size(op, dt, N, d_in, d_out, K) for op in range(3))
        self.ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        self.dloss = torch.empty((K, N), dtype=torch.float32, device=device)
        self.r = torch.empty((K, N), dtype=torch.float32, device=device)
        self.G_W = torch.empty((d_out, d_in), dtype=torch.float32, device=device)

    def estimate(self, x, W, u, cu_seqlens, sigma: float, gamma: float, key: NoiseKey,
                 stream=None):
        dust_noisy_linear_fwd(x, W, u, self.K, sigma, key, self.dloss, self.ws, stream)
        dust_credit(self.dloss, cu_seqlens, gamma, self.r, self.ws, stream)
        dust_weight_grad(self.r, x, self.d_out, self.K, sigma, key, self.G_W, False, None,
                         self.ws, stream)
        return self.G_W

    def estimate_from_host(self, hx, hW, hu, cu_seqlens, sigma: float, gamma: float,
                           key: NoiseKey, G_host=None, chunks: int = 4, reduce=None):
        """The estimate from inputs in pinned host memory, with the upload overlapped: the
        tokens are cut into ``chunks`` runs of whole sequences; each run is copied on a copy
        stream while the previous one goes through the forward, the credit and the weight
        estimate (accumulated over the runs, token offsets keeping the noise of the whole
        batch).  ``reduce`` (optional) is applied to the device G_W before it is copied back
        (for instance the all-reduce over data-parallel ranks).  G_W comes back into
        ``G_host`` (pinned, allocated if None).  Synchronises."""
        import numpy as np
        torch = _torch()
        dev = self.ws.device
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        N = int(cu[-1])
        if N != self.N:
            raise ValueError("cu_seqlens does not cover the layer's N tokens")
        if not hasattr(self, "_x"):
            self._x = torch.empty((N, self.d_in), dtype=hx.dtype, device=dev)
            self._u = torch.empty((N, self.d_out), dtype=hu.dtype, device=dev)
            self._W = torch.empty((self.d_out, self.d_in), dtype=hW.dtype, device=dev)
            self._copy = torch.cuda.Stream(device=dev)
        # cuts at sequence ends that keep the per-run views 16-byte aligned
        cuts = _sequence_cuts(cu, N, chunks)
        # every run's local cu_seqlens, uploaded once
        locs = [(cu[(cu >= a) & (cu <= b)] - a).astype(np.int32) for a, b in zip(cuts[:-1], cuts[1:])]
        cu_all = torch.from_numpy(np.concatenate(locs)).pin_memory().to(dev, non_blocking=True)
        offs = np.cumsum([0] + [len(l) for l in locs])
        comp = torch.cuda.current_stream(dev)
        ready = []
        self._copy.wait_stream(comp)  # the uploads start after the work already queued
        with torch.cuda.stream(self._copy):
            self._W.copy_(hW, non_blocking=True)
            for a, b in zip(cuts[:-1], cuts[1:]):
                self._x[a:b].copy_(hx[a:b], non_blocking=True)
                self._u[a:b].copy_(hu[a:b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self._copy)
                ready.append(ev)
        for n, ((a, b), ev) in enumerate(zip(zip(cuts[:-1], cuts[1:]), ready)):
            comp.wait_event(ev)
            cu_d = cu_all[int(offs[n]):int(offs[n + 1])]
            k = key._replace(token_offset=key.token_offset + a)
            x, u = self._x[a:b], self._u[a:b]
            dl, r = self.dloss[:, a:b], self.r[:, a:b]
            dust_noisy_linear_fwd(x, self._W, u, self.K, sigma, k, dl, self.ws)
            dust_credit(dl, cu_d, gamma, r, self.ws)
            dust_weight_grad(r, x, self.d_out, self.K, sigma, k, self.G_W, n > 0, None, self.ws)
        if reduce is not None:
            reduce(self.G_W)
        if G_host is None:
            G_host = torch.empty(self.G_W.shape, dtype=self.G_W.dtype, pin_memory=True)
        G_host.copy_(self.G_W, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()
        return G_host
