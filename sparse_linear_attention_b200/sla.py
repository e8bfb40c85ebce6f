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
SLA_FLAG_PREPARED, SLA_FLAG_FP8, SLA_FLAG_INT8, SLA_FLAG_WAIT_TEST = 1, 2, 4, 8
SLA_WS_FP8 = 0x100

STATUS_NAMES = {0: "SLA_OK", 1: "SLA_ERR_INVALID_ARG", 2: "SLA_ERR_UNSUPPORTED", 3: "SLA_ERR_ALIGNMENT",
                4: "SLA_ERR_WORKSPACE", 5: "SLA_ERR_CUDA", 6: "SLA_ERR_TIMEOUT", 7: "SLA_ERR_DEVICE_INDEX"}

EXPORTS = ("sla_status_string", "sla_last_error_detail", "sla_keep_count", "sla_workspace_size",
           "sla_workspace_init", "sla_route", "sla_route_noalloc", "sla_route_soft", "sla_prepare", "sla2_attn_fwd",
           "sla_attn_fwd", "sla2_attn_bwd_workspace_size", "sla2_attn_bwd", "sla_attn_bwd_workspace_size", "sla_attn_bwd",
           "sla2_forward_host_device_bytes", "sla2_forward_host", "sla_read_device_status")


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
        "sla_attn_bwd_workspace_size": (sz, [sp]),
        "sla_attn_bwd": (i, [sp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sla2_forward_host_device_bytes": (sz, [sp, i, i, u]),
        "sla2_forward_host": (i, [sp, vp, vp, vp, vp, vp, vp, i, i, u, vp, i, vp, vp, sz, vp]),
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


_IN_DTYPES = {SLA_F32: torch.float32, SLA_BF16: torch.bfloat16}


class _Args:
    """Checks, before a C call, that every tensor argument is where and what
    the C ABI expects: a contiguous CUDA tensor on the same device as the
    others, of the expected dtype and shape.  The C side only sees raw
    pointers, so a CPU, strided or wrongly shaped tensor must stop here."""

    def __init__(self, fn: str, shape: Shape):
        self.fn, self.dev = fn, None
        self.B, self.H, self.N, self.d = shape.B, shape.H, shape.N, shape.d
        self.nq = -(-shape.N // shape.bq) if shape.bq > 0 else 0
        self.nkv = -(-shape.N // shape.bkv) if shape.bkv > 0 else 0
        self.in_dtype = _IN_DTYPES.get(shape.in_dtype)

    def __call__(self, name, t, dims=None, dtypes=None, optional=False):
        if t is None:
            if optional:
                return
            raise ValueError(f"{self.fn}: {name} is required")
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{self.fn}: {name} must be a torch tensor, not {type(t).__name__}")
        if t.device.type != "cuda":
            raise ValueError(f"{self.fn}: {name} must be a CUDA tensor (got {t.device})")
        if self.dev is None:
            self.dev = t.device
        elif t.device != self.dev:
            raise ValueError(f"{self.fn}: {name} is on {t.device}, the other arguments on {self.dev}")
        if not t.is_contiguous():
            raise ValueError(f"{self.fn}: {name} must be contiguous")
        if dtypes is not None and t.dtype not in dtypes:
            raise TypeError(f"{self.fn}: {name} has dtype {t.dtype}, expected one of {list(dtypes)}")
        if dims is not None and tuple(t.shape) != tuple(dims):
            raise ValueError(f"{self.fn}: {name} has shape {tuple(t.shape)}, expected {tuple(dims)}")

    def qkv(self, **named):
        if self.in_dtype is None:
            raise ValueError(f"{self.fn}: shape.in_dtype must be SLA_F32 or SLA_BF16")
        for name, t in named.items():
            self(name, t, (self.B, self.H, self.N, self.d), (self.in_dtype,))

    def ws(self, t):
        self("ws", t)
        return t.numel() * t.element_size()


def _wmat(a, name, t, dtype):
    a(name, t, (a.d, a.d), (dtype,), optional=True)


def make_shape(q: torch.Tensor, bq: int, bkv: int = 64) -> Shape:
    B, H, N, d = q.shape
    return Shape(B, H, N, d, bq, bkv, _dtype_code(q))


def sla_keep_count(ratio: float, n_kv: int) -> int:
    return lib().sla_keep_count(float(ratio), int(n_kv))


def sla_workspace_size(shape: Shape, mode: int = SLA_MODE_SLA2_TOPK) -> int:
    return lib().sla_workspace_size(ctypes.byref(shape), mode)


def sla_workspace_init(ws: torch.Tensor, stream=None) -> None:
    nb = _Args("sla_workspace_init", Shape()).ws(ws)
    _check("sla_workspace_init", lib().sla_workspace_init(_p(ws), nb, _s(stream)))


def _route_outputs(a, k_keep, kept_idx, labels, scores_dbg):
    a("kept_idx", kept_idx, (a.B, a.H, a.nq, k_keep), (torch.int32,), optional=k_keep == 0)
    a("labels", labels, (a.B, a.H, a.nq, a.nkv), (torch.int8,), optional=True)
    a("scores_dbg", scores_dbg, (a.B, a.H, a.nq, a.nkv), (torch.float32,), optional=True)


def sla_route(shape: Shape, q, k, wq, wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, ws, stream=None):
    a = _Args("sla_route", shape)
    a.qkv(q=q, k=k)
    _wmat(a, "wq", wq, torch.float32)
    _wmat(a, "wk", wk, torch.float32)
    _route_outputs(a, k_keep, kept_idx, labels, scores_dbg)
    nb = a.ws(ws)
    _check("sla_route", lib().sla_route(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), mode, k_keep, k_neg,
                                        _p(kept_idx), _p(labels), _p(scores_dbg), _p(ws), nb, _s(stream)))


def sla_route_noalloc(shape: Shape, q, k, wq, wk, mode, k_keep, k_neg, kept_idx, labels, scores_dbg, stream=None):
    a = _Args("sla_route_noalloc", shape)
    a.qkv(q=q, k=k)
    _wmat(a, "wq", wq, torch.float32)
    _wmat(a, "wk", wk, torch.float32)
    _route_outputs(a, k_keep, kept_idx, labels, scores_dbg)
    _check("sla_route_noalloc", lib().sla_route_noalloc(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), mode,
                                                        k_keep, k_neg, _p(kept_idx), _p(labels), _p(scores_dbg),
                                                        _s(stream)))


def sla_route_soft(shape: Shape, q, k, wq, wk, k_keep, tau, mask, lam, ws, stream=None):
    a = _Args("sla_route_soft", shape)
    a.qkv(q=q, k=k)
    _wmat(a, "wq", wq, torch.float32)
    _wmat(a, "wk", wk, torch.float32)
    a("mask", mask, (a.B, a.H, a.nq, a.nkv), (torch.float32,))
    a("lambda", lam, (a.B, a.H, a.nq), (torch.float32,), optional=True)
    nb = a.ws(ws)
    _check("sla_route_soft", lib().sla_route_soft(ctypes.byref(shape), _p(q), _p(k), _p(wq), _p(wk), k_keep,
                                                  float(tau), _p(mask), _p(lam), _p(ws), nb, _s(stream)))


def sla_prepare(shape: Shape, k, v, phi, ws, stream=None):
    a = _Args("sla_prepare", shape)
    a.qkv(k=k, v=v)
    nb = a.ws(ws)
    _check("sla_prepare", lib().sla_prepare(ctypes.byref(shape), _p(k), _p(v), phi, _p(ws), nb, _s(stream)))


def sla2_attn_fwd(shape: Shape, q, k, v, kept_idx, k_keep, alpha, phi, flags, out, ws, stream=None):
    a = _Args("sla2_attn_fwd", shape)
    a.qkv(q=q, k=k, v=v)
    a("kept_idx", kept_idx, (a.B, a.H, a.nq, k_keep), (torch.int32,), optional=k_keep == 0)
    a("alpha", alpha, (a.B, a.H, a.nq), (torch.float32,))
    a("out", out, (a.B, a.H, a.N, a.d), (torch.float32, torch.bfloat16))
    nb = a.ws(ws)
    out_dt = _dtype_code(out)
    _check("sla2_attn_fwd", lib().sla2_attn_fwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(kept_idx), k_keep,
                                                _p(alpha), phi, flags, _p(out), out_dt, _p(ws), nb, _s(stream)))


def sla_attn_fwd(shape: Shape, q, k, v, labels, wproj, phi, flags, out, ws, stream=None):
    a = _Args("sla_attn_fwd", shape)
    a.qkv(q=q, k=k, v=v)
    a("labels", labels, (a.B, a.H, a.nq, a.nkv), (torch.int8,))
    a("wproj", wproj, (a.d, a.d), (torch.bfloat16,))
    a("out", out, (a.B, a.H, a.N, a.d), (torch.float32, torch.bfloat16))
    nb = a.ws(ws)
    out_dt = _dtype_code(out)
    _check("sla_attn_fwd", lib().sla_attn_fwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(labels), _p(wproj), phi,
                                              flags, _p(out), out_dt, _p(ws), nb, _s(stream)))


def sla2_attn_bwd_workspace_size(shape: Shape) -> int:
    return lib().sla2_attn_bwd_workspace_size(ctypes.byref(shape))


def sla2_attn_bwd(shape: Shape, q, k, v, kept_idx, k_keep, alpha, phi, dout, dq, dk, dv, dalpha, ws, stream=None):
    a = _Args("sla2_attn_bwd", shape)
    a.qkv(q=q, k=k, v=v, dout=dout)
    a("kept_idx", kept_idx, (a.B, a.H, a.nq, k_keep), (torch.int32,), optional=k_keep == 0)
    a("alpha", alpha, (a.B, a.H, a.nq), (torch.float32,))
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        a(name, t, (a.B, a.H, a.N, a.d), (torch.float32,))
    a("dalpha", dalpha, (a.B, a.H, a.nq), (torch.float32,))
    nb = a.ws(ws)
    _check("sla2_attn_bwd", lib().sla2_attn_bwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(kept_idx), k_keep,
                                                _p(alpha), phi, _p(dout), _p(dq), _p(dk), _p(dv), _p(dalpha),
                                                _p(ws), nb, _s(stream)))


def sla_attn_bwd_workspace_size(shape: Shape) -> int:
    return lib().sla_attn_bwd_workspace_size(ctypes.byref(shape))


def sla_attn_bwd(shape: Shape, q, k, v, labels, wproj, phi, dout, dq, dk, dv, dwproj, ws, stream=None):
    a = _Args("sla_attn_bwd", shape)
    a.qkv(q=q, k=k, v=v, dout=dout)
    a("labels", labels, (a.B, a.H, a.nq, a.nkv), (torch.int8,))
    a("wproj", wproj, (a.d, a.d), (torch.bfloat16,))
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        a(name, t, (a.B, a.H, a.N, a.d), (torch.float32,))
    a("dwproj", dwproj, (a.d, a.d), (torch.float32,))
    nb = a.ws(ws)
    _check("sla_attn_bwd", lib().sla_attn_bwd(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(labels), _p(wproj), phi,
                                              _p(dout), _p(dq), _p(dk), _p(dv), _p(dwproj), _p(ws), nb, _s(stream)))


def sla2_forward_host_device_bytes(shape: Shape, k_keep: int, out_dtype: int = SLA_BF16, flags: int = 0) -> int:
    return lib().sla2_forward_host_device_bytes(ctypes.byref(shape), int(k_keep), int(out_dtype), int(flags))


def _host(a, name, t, dims, dtypes, optional=False):
    """A host-side argument of sla2_forward_host: a contiguous CPU tensor."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{a.fn}: {name} is required")
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise ValueError(f"{a.fn}: {name} must be a CPU (host) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{a.fn}: {name} must be contiguous")
    if t.dtype not in dtypes:
        raise TypeError(f"{a.fn}: {name} has dtype {t.dtype}, expected one of {list(dtypes)}")
    if tuple(t.shape) != tuple(dims):
        raise ValueError(f"{a.fn}: {name} has shape {tuple(t.shape)}, expected {tuple(dims)}")


def sla2_forward_host(shape: Shape, q, k, v, wq, wk, alpha, k_keep, phi, flags, out, kept_out, dev, stream=None):
    """Host tensors in (pin them for asynchronous copies), host out; `dev` a
    CUDA byte buffer of sla2_forward_host_device_bytes bytes."""
    a = _Args("sla2_forward_host", shape)
    if a.in_dtype is None:
        raise ValueError("sla2_forward_host: shape.in_dtype must be SLA_F32 or SLA_BF16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _host(a, name, t, (a.B, a.H, a.N, a.d), (a.in_dtype,))
    _host(a, "wq", wq, (a.d, a.d), (torch.float32,), optional=True)
    _host(a, "wk", wk, (a.d, a.d), (torch.float32,), optional=True)
    _host(a, "alpha", alpha, (a.B, a.H, a.nq), (torch.float32,))
    _host(a, "out", out, (a.B, a.H, a.N, a.d), (torch.float32, torch.bfloat16))
    _host(a, "kept_out", kept_out, (a.B, a.H, a.nq, k_keep), (torch.int32,), optional=True)
    nb = a.ws(dev)
    _check("sla2_forward_host", lib().sla2_forward_host(ctypes.byref(shape), _p(q), _p(k), _p(v), _p(wq), _p(wk),
                                                        _p(alpha), k_keep, phi, flags, _p(out), _dtype_code(out),
                                                        _p(kept_out), _p(dev), nb, _s(stream)))


def sla_read_device_status(ws, stream=None) -> int:
    _Args("sla_read_device_status", Shape())("ws", ws)
    return lib().sla_read_device_status(_p(ws), _s(stream))
