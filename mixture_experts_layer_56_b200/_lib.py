"""ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every function below has the name of the C entry point it calls; tensors are
passed as device (or host) pointers, ``None`` as NULL, and the stream defaults
to torch's current CUDA stream.  A non-zero status raises ``MoeError``.
Loading fails loudly when the library has not been built: there is no other
implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_int, c_int32, c_int64, c_size_t, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_DTYPE_F32 = 0
MOE_DTYPE_BF16 = 1
MOE_FLAG_BIAS_SELECT_ONLY = 1
MOE_FLAG_GEMM_SINGLE_CTA = 2
MOE_FLAG_GEMM_CTA_PAIR = 4
MOE_FLAG_ROUTER_SIMT = 8
MOE_FLAG_INJECT_WAIT_TIMEOUT = 16
MOE_FLAG_GEMM_NARROW = 32

MOE_OK = 0
MOE_ERR_NULLPTR = -1
MOE_ERR_SHAPE = -2
MOE_ERR_ALIGN = -3
MOE_ERR_WORKSPACE = -4
MOE_ERR_DTYPE = -5
MOE_ERR_CUDA = -6
MOE_ERR_DEVICE_CHECK = -7
MOE_ERR_UNSUPPORTED = -8
MOE_ERR_SCRATCH_LIMIT = -9

# stage kinds of the tracer (include/moe.h MOE_KERNEL_*)
MOE_KERNEL_ROUTER = 1
MOE_KERNEL_DISPATCH = 2
MOE_KERNEL_GATHER = 3
MOE_KERNEL_GEMM_GATE_UP = 4
MOE_KERNEL_GEMM_DOWN = 5
MOE_KERNEL_COMBINE = 6
MOE_KERNEL_FFN_F32 = 7
MOE_KERNEL_MEMSET = 8
MOE_KERNEL_PACK = 9
MOE_KERNEL_BALANCE = 10
MOE_KERNEL_DECODE_LAYER = 11
MOE_PATH_STAGES = 0
MOE_PATH_DECODE_LAYER = 1
MOE_PATH_SMALL_BATCH = 2
MOE_DISPATCH_STATIC_SCRATCH_BYTES = 512 * 1024


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({strerror(code)})")


class MoeShape(ctypes.Structure):
    _fields_ = [("T", c_int64), ("d", c_int32), ("n_routed", c_int32), ("n_shared", c_int32),
                ("inter", c_int32), ("top_k", c_int32), ("dtype", c_int32), ("flags", c_int32)]

    def __repr__(self):
        return (f"MoeShape(T={self.T}, d={self.d}, n_routed={self.n_routed}, "
                f"n_shared={self.n_shared}, inter={self.inter}, top_k={self.top_k}, "
                f"dtype={self.dtype}, flags={self.flags})")


_SHAPE = POINTER(MoeShape)
_V = c_void_p

# name -> (restype, argtypes)
SIGNATURES = {
    "moe_strerror": (c_char_p, [c_int]),
    "moe_version": (c_char_p, []),
    "moe_launch_count": (c_uint64, []),
    "moe_workspace_size": (c_int, [_SHAPE, POINTER(c_size_t)]),
    "moe_workspace_size_host": (c_int, [_SHAPE, POINTER(c_size_t)]),
    "moe_forward_path": (c_int, [_SHAPE, POINTER(c_int32)]),
    "moe_pack_w13": (c_int, [_SHAPE, c_int32, _V, _V, _V, _V]),
    "moe_route": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V]),
    "moe_dispatch": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, c_size_t, _V]),
    "moe_dispatch_static_scratch": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V]),
    "moe_expert_ffn": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, c_size_t, _V]),
    "moe_combine": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, _V]),
    "moe_layer_forward": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, _V, _V, _V, c_size_t, _V]),
    "moe_layer_forward_host": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, _V, _V, _V, c_size_t, _V]),
    "moe_expert_balance": (c_int, [_SHAPE, _V, _V, _V, _V, _V, _V, _V, c_size_t, _V]),
    "moe_read_status": (c_int, [_V, POINTER(c_int32), _V]),
    "moe_profile_enable": (c_int, [c_int]),
    "moe_profile_read": (c_int, [POINTER(c_int32), POINTER(ctypes.c_float), c_int32,
                                 POINTER(c_int32)]),
    "moe_kernel_name": (c_char_p, [c_int32]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if libmoe.so is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mixture_experts_layer_56_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def strerror(code: int) -> str:
    return lib().moe_strerror(code).decode()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, rc):
    if rc != MOE_OK:
        raise MoeError(fn, rc)
    return rc


def make_shape(T, d, n_routed, n_shared, inter, top_k, dtype=MOE_DTYPE_BF16, flags=0) -> MoeShape:
    return MoeShape(T, d, n_routed, n_shared, inter, top_k, dtype, flags)


# ------------------------------------------------------------- entry points
def moe_version() -> str:
    return lib().moe_version().decode()


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


def moe_workspace_size(shape: MoeShape) -> int:
    n = c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def moe_workspace_size_host(shape: MoeShape) -> int:
    n = c_size_t(0)
    _check("moe_workspace_size_host",
           lib().moe_workspace_size_host(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def moe_forward_path(shape: MoeShape) -> int:
    p = c_int32(0)
    _check("moe_forward_path", lib().moe_forward_path(ctypes.byref(shape), ctypes.byref(p)))
    return p.value


def moe_pack_w13(shape, n_experts, W1, W3, W13, stream=None):
    return _check("moe_pack_w13", lib().moe_pack_w13(
        ctypes.byref(shape), n_experts, _ptr(W1), _ptr(W3), _ptr(W13), _stream(stream)))


def moe_route(shape, u, E, bias, idx, w, stream=None):
    return _check("moe_route", lib().moe_route(
        ctypes.byref(shape), _ptr(u), _ptr(E), _ptr(bias), _ptr(idx), _ptr(w), _stream(stream)))


def moe_dispatch(shape, idx, counts, offsets, perm, inv, ws, ws_bytes=None, stream=None):
    nb = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return _check("moe_dispatch", lib().moe_dispatch(
        ctypes.byref(shape), _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
        _ptr(ws), nb, _stream(stream)))


def moe_dispatch_static_scratch(shape, idx, counts, offsets, perm, inv, stream=None):
    return _check("moe_dispatch_static_scratch", lib().moe_dispatch_static_scratch(
        ctypes.byref(shape), _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv),
        _stream(stream)))


def moe_expert_ffn(shape, u, perm, offsets, W13, W2, W13_s, W2_s, y, ysh, ws, ws_bytes=None,
                   stream=None):
    nb = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(shape), _ptr(u), _ptr(perm), _ptr(offsets), _ptr(W13), _ptr(W2),
        _ptr(W13_s), _ptr(W2_s), _ptr(y), _ptr(ysh), _ptr(ws), nb, _stream(stream)))


def moe_combine(shape, u, ysh, y, w, inv, h, stream=None):
    return _check("moe_combine", lib().moe_combine(
        ctypes.byref(shape), _ptr(u), _ptr(ysh), _ptr(y), _ptr(w), _ptr(inv), _ptr(h),
        _stream(stream)))


def moe_layer_forward(shape, u, E, bias, W13, W2, W13_s, W2_s, h, ws, ws_bytes=None,
                      stream=None):
    nb = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(shape), _ptr(u), _ptr(E), _ptr(bias), _ptr(W13), _ptr(W2), _ptr(W13_s),
        _ptr(W2_s), _ptr(h), _ptr(ws), nb, _stream(stream)))


def moe_layer_forward_host(shape, u_host, E, bias, W13, W2, W13_s, W2_s, h_host, ws,
                           ws_bytes=None, stream=None):
    nb = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return _check("moe_layer_forward_host", lib().moe_layer_forward_host(
        ctypes.byref(shape), _ptr(u_host), _ptr(E), _ptr(bias), _ptr(W13), _ptr(W2),
        _ptr(W13_s), _ptr(W2_s), _ptr(h_host), _ptr(ws), nb, _stream(stream)))


def moe_expert_balance(shape, u, E, bias, counts, f, P, ws, ws_bytes=None, stream=None):
    nb = ws.numel() * ws.element_size() if ws_bytes is None else ws_bytes
    return _check("moe_expert_balance", lib().moe_expert_balance(
        ctypes.byref(shape), _ptr(u), _ptr(E), _ptr(bias), _ptr(counts), _ptr(f), _ptr(P),
        _ptr(ws), nb, _stream(stream)))


def moe_read_status(ws, stream=None) -> int:
    st = c_int32(0)
    _check("moe_read_status", lib().moe_read_status(_ptr(ws), ctypes.byref(st), _stream(stream)))
    return st.value


def moe_profile_enable(on=True, kinds=None):
    """Turn stage tracing on or off; `kinds` (MOE_KERNEL_* values) limits it
    to those stages."""
    if not on:
        v = 0
    elif kinds is None:
        v = 1
    else:
        v = 0
        for k in kinds:
            v |= 1 << int(k)
    return _check("moe_profile_enable", lib().moe_profile_enable(v))


def moe_profile_read(max_entries: int = 4096):
    """[(stage name, milliseconds), ...] since the last read (synchronises)."""
    kinds = (c_int32 * max_entries)()
    ms = (ctypes.c_float * max_entries)()
    n = c_int32(0)
    _check("moe_profile_read", lib().moe_profile_read(kinds, ms, max_entries, ctypes.byref(n)))
    return [(moe_kernel_name(kinds[i]), float(ms[i])) for i in range(n.value)]


def moe_kernel_name(kind: int) -> str:
    return lib().moe_kernel_name(kind).decode()
