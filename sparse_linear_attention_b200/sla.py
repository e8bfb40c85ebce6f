"""Python binding of libsla (include/sla.h): argument marshalling only.

Every function has the name of the C entry point it calls.  Tensors are torch
CUDA tensors (the caller allocates them); streams default to torch's current
stream.  All computation happens in libsla's CUDA kernels: there is no Python
or CPU fallback, and a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsla.so")

SLA_OK = 0
SLA_F32, SLA_BF16 = 0, 1
SLA_PHI_ELU1, SLA_PHI_SOFTMAX = 0, 1
SLA_MODE_SLA2_TOPK, SLA_MODE_SLA_3WAY = 0, 1
SLA_ROUTE_KBAR_FROM_WS = 0x10
SLA_FLAG_PREPARED, SLA_FLAG_FP8 = 1, 2
SLA_WS_FP8 = 0x100

STATUS_NAMES = {0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_ALIGNMENT",
                4: "SLA_ERR_WORKSPACE", 5: "SLA_ERR_CUDA", 6: "SLA_ERR_TIMEOUT", 7: "SLA_ERR_DEVICE_INDEX"}

EXPORTS = ("sla_status_string", "sla_last_error_detail", "sla_keep_count", "sla_workspace_size",
           "sla_workspace_init", "sla_route", "sla_route_noalloc", "sla_route_soft", "sla_prepare", "sla2_attn_fwd",
           "sla_attn_fwd", "sla2_attn_bwd_workspace_size", "sla2_attn_bwd",
           "sla_read_device_status")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("bq", ctypes.c_int), ("bkv", ctypes.c_int), ("in_dtype", ctypes.c_int)]


class SLAError(RuntimeError):
    def __init__(self, fn, status, detail):
        self.status = status
        super().__init__(f"{fn} -> {STATUS_NAMES.get(status, status)}: {detail}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsla.so from the package directory (built by __graft_entry__.build())."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libsla.so not found at {LIB_PATH}; build it with "
                          f"`python -m sparse_linear_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint
    sp = ctypes.POINTER(Shape)
    sig = {
        "sla_status_string": (ctypes.c_char_p, [i]),
        "sla_last_error_detail": (ctypes.c_char_p, []),
        "sla_keep_count": (i, [ctypes.c_double, i]),
        "sla_workspace_size": (sz, [sp, i]),
        "sla_workspace_init": (i, [vp, sz, vp]),
        "sla_route": (i, [sp, vp, vp, vp, vp, i, i, i, vp, vp, vp, vp, sz, vp]),
        "sla_route_noalloc": (i, [sp, vp, vp, vp, vp, i, i, i, vp, vp, vp, vp]),
        "sla_route_soft": (i, [sp, vp, vp, vp, vp, i, ctypes.c_float, vp, vp, vp, sz, vp]),
        "sla_prepare": (i, [sp, vp, vp, i, vp, sz, vp]),
        "sla2_attn_fwd": (i, [sp, vp, vp, vp, vp, i, vp, i, u, vp, i, vp, sz, vp]),
        "sla_attn_fwd": (i, [sp, vp, vp, vp, vp, vp, i, u, vp, i, vp, sz, vp]),
        "sla2_attn_bwd_workspace_size": (sz, [sp]),
        "sla2_attn_bwd": (i, [sp, vp, vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sla_read_device_status": (i, [vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(fn, status):
    if status != SLA_OK:
        detail = lib().sla_last_error_detail().decode()
        raise SLAError(fn, status, detail)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SLA_BF16
    if t.dtype == torch.float32:
        return SLA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_shape(q: torch.Tensor, bq: int, bkv: int = 64) -> Shape:
    B, H, N, d = q.shape
    return Shape(B, H, N, d, bq, bkv, _dtype_code(q))


def sla_keep_count(ratio: float, n_kv: int) -> int:
    return lib().sla_keep_count(float(ratio), int(n_kv))


def sla_workspace_size(shape: Shape, mode: int = SLA_MODE_SLA2_TOPK) -> int:
    return lib().sla_workspace_size(ctypes.byref(shape), mode)


def sla_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check("sla_workspace_init", lib().sla_workspace_init(_p(ws), ws.numel(), _s(stream)))


def sla_route(shape: Shape, q, k, wq, wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, ws, stream=None):
    _check("sla_route", lib().sla_route(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), mode, k_keep, k_neg,
                                        _p(kept_idx), _p(labels), _p(scores_dbg), _p(ws), ws.numel(), _s(stream)))


def sla_route_noalloc(shape: Shape, q, k, wq, wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, stream=None):
    _check("sla_route_noalloc", lib().sla_route_noalloc(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), mode,
                                                        k_keep, k_neg, _p(kept_idx), _p(labels), _p(scores_dbg),
                                                        _s(stream)))


def sla_route_soft(shape: Shape, q, k, wq, wk, k_keep, tau, mask, lam, ws, stream=None):
    _check("sla_route_soft", lib().sla_route_soft(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), k_keep,
                                                  float(tau), _p(mask), _p(lam), _p(ws), ws.numel(), _s(stream)))


def sla_prepare(shape: Shape, k, v, phi, ws, stream=None):
    _check("sla_prepare", lib().sla_prepare(ctypes.byref(shape), _p(k), _p(v), phi, _p(ws), ws.numel(), _s(stream)))


def sla2_attn_fwd(shape: Shape, q, k, v, kept_idx, k_keep, alpha, phi, flags, out, ws, stream=None):
    out_dt = _dtype_code(out)
    _check("sla2_attn_fwd", lib().sla2_attn_fwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(kept_idx), k_keep,
                                                _p(alpha), phi, flags, _p(out), out_dt, _p(ws), ws.numel(),
                                                _s(stream)))


def sla_attn_fwd(shape: Shape, q, k, v, labels, wproj, phi, flags, out, ws, stream=None):
    out_dt = _dtype_code(out)
    _check("sla_attn_fwd", lib().sla_attn_fwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(labels), _p(wproj), phi,
                                              flags, _p(out), out_dt, _p(ws), ws.numel(), _s(stream)))


def sla2_attn_bwd_workspace_size(shape: Shape) -> int:
    return lib().sla2_attn_bwd_workspace_size(ctypes.byref(shape))


def sla2_attn_bwd(shape: Shape, q, k, v, kept_idx, k_keep, alpha, phi, dout, dq, dk, dv, dalpha, ws, stream=None):
    _check("sla2_attn_bwd", lib().sla2_attn_bwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(kept_idx), k_keep,
                                                _p(alpha), phi, _p(dout), _p(dq), _p(dk), _p(dv), _p(dalpha),
                                                _p(ws), ws.numel(), _s(stream)))


def sla_read_device_status(ws, stream=None) -> int:
    return lib().sla_read_device_status(_p(ws), _s(stream))
