"""ctypes binding of libqsm.so (declared in include/qsm.h).

The functions named like the C entry points (``qsm_attn_fwd``, ...) marshal
torch tensors into pointers and sizes and call the library; every step of the
computation runs in the library's CUDA kernels.  PyTorch only provides device
memory and the current stream.  There is no fallback: if the library is
missing, or a tensor is not on a CUDA device, the call raises.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsm.so")

# enums of include/qsm.h
QSM_OK, QSM_ERR_INVALID_ARG, QSM_ERR_UNSUPPORTED, QSM_ERR_CUDA, QSM_ERR_TIMEOUT = range(5)
MODE_EXACT, MODE_KINTERVAL, MODE_ROWMAX_POT, MODE_TRUNCATED, MODE_UNIFORM = 0, 1, 2, 3, 4
CALIB_MINMAX, CALIB_FIXED_WINDOW = 0, 1
ROUND_INTERP, ROUND_HARD = 0, 1
SURR_NONE, SURR_PRE, SURR_POST = 0, 1, 2
DTYPE_BF16, DTYPE_FP8_E4M3 = 0, 1
ANCHOR_FINAL, ANCHOR_RUNNING = 0, 1

EXPORTED = ("qsm_opts_default", "qsm_attn_fwd", "qsm_attn_bwd", "qsm_attn_bwd_workspace_size",
            "qsm_attn_bwd_noalloc", "qsm_weight_map", "qsm_status_string", "qsm_version")
NOALLOC_SCRATCH_BYTES = 16 << 20     # QSM_NOALLOC_SCRATCH_BYTES


class QsmOpts(ctypes.Structure):
    """Mirror of ``qsm_opts``."""
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("q_descale", ctypes.c_float),
        ("k_descale", ctypes.c_float),
        ("v_descale", ctypes.c_float),
        ("window", ctypes.c_float),
        ("pot_floor", ctypes.c_int),
        ("below_policy", ctypes.c_int),
        ("detach_extrema", ctypes.c_int),
        ("row_hi", ctypes.c_void_p),
        ("row_lo", ctypes.c_void_p),
        ("row_argmax", ctypes.c_void_p),
        ("row_argmin", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("status_dev", ctypes.c_void_p),
        ("debug_idx", ctypes.c_void_p),
        ("debug_flags", ctypes.c_int),
        ("anchor", ctypes.c_int),
        ("support", ctypes.c_float),
    ]


class QsmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, qsm_status_string(status)))


_lib = None


def lib():
    """Load libqsm.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libqsm.so not found at %s: build it with "
                           "`python -m approximate_softmax_attention_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.qsm_opts_default.argtypes = [ctypes.POINTER(QsmOpts)]
    L.qsm_opts_default.restype = None
    L.qsm_attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci,
                               ctypes.POINTER(QsmOpts), vp]
    L.qsm_attn_fwd.restype = ci
    L.qsm_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                               ci, ci, ci, ctypes.POINTER(QsmOpts), vp]
    L.qsm_attn_bwd.restype = ci
    L.qsm_attn_bwd_noalloc.argtypes = list(L.qsm_attn_bwd.argtypes)
    L.qsm_attn_bwd_noalloc.restype = ci
    L.qsm_attn_bwd_workspace_size.argtypes = [ci, ci, ci, ci]
    L.qsm_attn_bwd_workspace_size.restype = ctypes.c_size_t
    L.qsm_weight_map.argtypes = [vp, vp, ci, ci, ci, ci, ci, ci, ctypes.POINTER(QsmOpts), vp, vp,
                                 vp, vp, vp]
    L.qsm_weight_map.restype = ci
    L.qsm_status_string.argtypes = [ci]
    L.qsm_status_string.restype = ctypes.c_char_p
    L.qsm_version.argtypes = []
    L.qsm_version.restype = ctypes.c_char_p
    _lib = L
    return L


def qsm_status_string(status: int) -> str:
    return lib().qsm_status_string(int(status)).decode()


def qsm_version() -> str:
    return lib().qsm_version().decode()


def qsm_opts_default() -> QsmOpts:
    o = QsmOpts()
    lib().qsm_opts_default(ctypes.byref(o))
    return o


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return int(t)
    if not t.is_cuda:
        raise ValueError("tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor is not contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_opts(**kw) -> QsmOpts:
    """qsm_opts with defaults, fields given as keywords (tensors -> pointers)."""
    o = qsm_opts_default()
    for k, v in kw.items():
        if isinstance(v, torch.Tensor):
            v = _ptr(v)
        setattr(o, k, v)
    return o


def qsm_attn_fwd(Q, K, V, O, LSE, causal, mode, Kint=4, calibration=CALIB_MINMAX,
                 rounding=ROUND_HARD, surrogate=SURR_NONE, opts=None, stream=None) -> int:
    B, H, S, D = Q.shape
    return lib().qsm_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, S, D,
                              int(causal), int(mode), int(Kint), int(calibration), int(rounding),
                              int(surrogate), ctypes.byref(opts) if opts is not None else None,
                              _stream(stream))


def qsm_attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, causal, mode, Kint=4,
                 calibration=CALIB_MINMAX, rounding=ROUND_HARD, surrogate=SURR_NONE, opts=None,
                 stream=None) -> int:
    B, H, S, D = Q.shape
    return lib().qsm_attn_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE), _ptr(dQ),
                              _ptr(dK), _ptr(dV), B, H, S, D, int(causal), int(mode), int(Kint),
                              int(calibration), int(rounding), int(surrogate),
                              ctypes.byref(opts) if opts is not None else None, _stream(stream))


def qsm_attn_bwd_noalloc(Q, K, V, O, dO, LSE, dQ, dK, dV, causal, mode, Kint=4,
                         calibration=CALIB_MINMAX, rounding=ROUND_HARD, surrogate=SURR_NONE,
                         opts=None, stream=None) -> int:
    """qsm_attn_bwd with the library's static scratch instead of a workspace
    (for callers that cannot allocate device memory at call time)."""
    B, H, S, D = Q.shape
    return lib().qsm_attn_bwd_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(LSE),
                                      _ptr(dQ), _ptr(dK), _ptr(dV), B, H, S, D, int(causal),
                                      int(mode), int(Kint), int(calibration), int(rounding),
                                      int(surrogate),
                                      ctypes.byref(opts) if opts is not None else None,
                                      _stream(stream))


def qsm_attn_bwd_workspace_size(B, H, S, D) -> int:
    return int(lib().qsm_attn_bwd_workspace_size(B, H, S, D))


def qsm_weight_map(scores, valid_len, mode, Kint=4, calibration=CALIB_MINMAX,
                   rounding=ROUND_HARD, opts=None, w=None, idx=None, hi=None, lo=None,
                   stream=None) -> int:
    rows, cols = scores.shape
    return lib().qsm_weight_map(_ptr(scores), _ptr(valid_len), rows, cols, int(mode), int(Kint),
                                int(calibration), int(rounding),
                                ctypes.byref(opts) if opts is not None else None, _ptr(w),
                                _ptr(idx), _ptr(hi), _ptr(lo), _stream(stream))


# ------------------------------------------------------------ convenience

def _check(status, where):
    if status != QSM_OK:
        raise QsmError(status, where)


def attention_forward(q, k, v, causal=False, mode=MODE_EXACT, Kint=4,
                      calibration=CALIB_MINMAX, rounding=ROUND_HARD, *, scale=None,
                      q_descale=1.0, k_descale=1.0, v_descale=1.0, window=8.0, pot_floor=15,
                      below_policy=0, stats=False, debug_idx=None, anchor=ANCHOR_FINAL,
                      support=4.0, stream=None):
    """Allocate the outputs with torch and run ``qsm_attn_fwd``.

    Returns (O, LSE) or (O, LSE, stats dict) with hi, lo, argmax, argmin
    (with ``anchor=ANCHOR_RUNNING``, the one-sweep form: hi and lo only).
    """
    B, H, S, D = q.shape
    dev = q.device
    O = torch.empty(B, H, S, D, dtype=torch.bfloat16, device=dev)
    LSE = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    st = None
    kw = dict(dtype=DTYPE_FP8_E4M3 if q.dtype == torch.float8_e4m3fn else DTYPE_BF16,
              scale=0.0 if scale is None else float(scale), q_descale=float(q_descale),
              k_descale=float(k_descale), v_descale=float(v_descale), window=float(window),
              pot_floor=int(pot_floor), below_policy=int(below_policy), anchor=int(anchor),
              support=float(support))
    if stats:
        st = dict(hi=torch.empty(B, H, S, dtype=torch.float32, device=dev),
                  lo=torch.empty(B, H, S, dtype=torch.float32, device=dev))
        kw.update(row_hi=st["hi"], row_lo=st["lo"])
        if anchor == ANCHOR_FINAL:
            st.update(argmax=torch.empty(B, H, S, dtype=torch.int32, device=dev),
                      argmin=torch.empty(B, H, S, dtype=torch.int32, device=dev))
            kw.update(row_argmax=st["argmax"], row_argmin=st["argmin"])
    if debug_idx is not None:
        kw["debug_idx"] = debug_idx
    opts = make_opts(**kw)
    _check(qsm_attn_fwd(q, k, v, O, LSE, causal, mode, Kint, calibration, rounding, SURR_NONE,
                        opts, stream), "qsm_attn_fwd")
    return (O, LSE, st) if stats else (O, LSE)


def default_scale(D):
    return 1.0 / math.sqrt(D)


def attention_backward(q, k, v, O, dO, LSE, stats, causal=False, mode=MODE_KINTERVAL, Kint=4,
                       calibration=CALIB_MINMAX, rounding=ROUND_HARD, surrogate=SURR_NONE, *,
                       detach_extrema=False, scale=None, q_descale=1.0, k_descale=1.0,
                       v_descale=1.0, window=8.0, below_policy=0, workspace=None, stream=None):
    """Allocate dQ, dK, dV (bf16; and the workspace, unless given) with torch
    and run ``qsm_attn_bwd``.  ``stats`` is the dict returned by
    attention_forward(..., stats=True).  With e4m3 q, k, v (and their
    descales, as given to the forward) the gradients are those of
    q_descale q, k_descale k, v_descale v."""
    B, H, S, D = q.shape
    dev = q.device
    dQ = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    dK = torch.empty(k.shape, dtype=torch.bfloat16, device=dev)
    dV = torch.empty(v.shape, dtype=torch.bfloat16, device=dev)
    need = qsm_attn_bwd_workspace_size(B, H, S, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    kw = dict(dtype=DTYPE_FP8_E4M3 if q.dtype == torch.float8_e4m3fn else DTYPE_BF16,
              scale=0.0 if scale is None else float(scale), q_descale=float(q_descale),
              k_descale=float(k_descale), v_descale=float(v_descale), window=float(window),
              below_policy=int(below_policy), detach_extrema=int(bool(detach_extrema)),
              workspace=workspace, workspace_bytes=int(workspace.numel()))
    if stats is not None:
        kw.update(row_hi=stats["hi"], row_lo=stats["lo"], row_argmax=stats["argmax"],
                  row_argmin=stats["argmin"])
    opts = make_opts(**kw)
    _check(qsm_attn_bwd(q, k, v, O, dO, LSE, dQ, dK, dV, causal, mode, Kint, calibration,
                        rounding, surrogate, opts, stream), "qsm_attn_bwd")
    return dQ, dK, dV
