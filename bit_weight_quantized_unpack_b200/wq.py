"""Python binding of libwq's C ABI (include/wq.h): argument marshalling only.

Each function has the name and argument order of its C counterpart. Tensor arguments are
torch tensors on the current CUDA device (their data_ptr() is passed) or raw integer
device pointers; `stream` defaults to torch's current stream. A non-zero wq_status is
raised as WQError. torch provides device memory and streams only: every step of the
computation runs in libwq's CUDA kernels, and there is no other implementation to fall
back to -- if libwq.so is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with "
                      "`python -m bit_weight_quantized_unpack_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

WQ_INT4, WQ_INT2, WQ_TERNARY, WQ_INT3, WQ_INT4H = 0, 1, 2, 3, 4
FMT = {"int4": WQ_INT4, "int2": WQ_INT2, "ternary": WQ_TERNARY, "int3": WQ_INT3, "int4h": WQ_INT4H}
WQ_OK, WQ_ERR_ARG, WQ_ERR_SHAPE, WQ_ERR_ALIGN, WQ_ERR_CUDA, WQ_ERR_UNSUPPORTED, WQ_ERR_SCRATCH = range(7)
WQ_ARGMAX_STATIC_SCRATCH_BYTES = 16384
WQ_LINEAR_SET_MAX = 256
WQ_RESCORE_MAX_TOPK = 64

_i64, _p, _i = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int


class wq_linear_desc(ctypes.Structure):
    _fields_ = [("codes", _p), ("scale", _p), ("zero", _p), ("x", _p), ("y", _p),
                ("N", _i64), ("K", _i64), ("M", _i64)]


_sig = {
    "wq_codes_bytes": (ctypes.c_size_t, [_i, _i64, _i64]),
    "wq_meta_count": (ctypes.c_size_t, [_i64, _i64]),
    "wq_scale_bytes": (ctypes.c_size_t, [_i, _i64, _i64]),
    "wq_zero_bytes": (ctypes.c_size_t, [_i, _i64, _i64]),
    "wq_quantize": (_i, [_p, _i64, _i64, _i, _i, _p, _p, _p, _p]),
    "wq_gemv": (_i, [_p, _p, _p, _p, _i, _i64, _i64, _p, _p]),
    "wq_gemm": (_i, [_p, _i64, _p, _p, _p, _i, _i64, _i64, _p, _p]),
    "wq_linear_set": (_i, [ctypes.POINTER(wq_linear_desc), _i, _i, _p]),
    "wq_status_str": (ctypes.c_char_p, [_i]),
    "wq_last_cuda_error": (_i, []),
    "wq_device_errors": (_i, [ctypes.POINTER(ctypes.c_uint), _i, _p]),
    "wq_debug_arm_timeout": (_i, [ctypes.c_uint]),
    "wq_argmax_workspace_bytes": (ctypes.c_size_t, []),
    "wq_gemv_argmax": (_i, [_p, _p, _p, _p, _i, _i64, _i64, _p, _p, _p, ctypes.c_size_t, _p]),
    "wq_gemv_argmax_static": (_i, [_p, _p, _p, _p, _i, _i64, _i64, _p, _p, _p]),
    "wq_rescore_workspace_bytes": (ctypes.c_size_t, [_i64, _i]),
    "wq_gemv_rescore": (_i, [_p, _p, _p, _p, _i, _p, _i64, _i64, _i, _p, _p, _p, _p, _p,
                             ctypes.c_size_t, _p]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class WQError(RuntimeError):
    def __init__(self, status: int, call: str):
        msg = _lib.wq_status_str(status).decode()
        if status == WQ_ERR_CUDA:
            msg += f" (cudaError {_lib.wq_last_cuda_error()})"
        super().__init__(f"{call}: {msg}")
        self.status = status


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _fmt(fmt):
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


def _check(status, call):
    if status != WQ_OK:
        raise WQError(status, call)


def wq_codes_bytes(fmt, N: int, K: int) -> int:
    return _lib.wq_codes_bytes(_fmt(fmt), N, K)


def wq_meta_count(N: int, K: int) -> int:
    return _lib.wq_meta_count(N, K)


def wq_scale_bytes(fmt, N: int, K: int) -> int:
    return _lib.wq_scale_bytes(_fmt(fmt), N, K)


def wq_zero_bytes(fmt, N: int, K: int) -> int:
    return _lib.wq_zero_bytes(_fmt(fmt), N, K)


def wq_quantize(W, N, K, fmt, group, codes, scale, zero, stream=None) -> None:
    _check(_lib.wq_quantize(_ptr(W), N, K, _fmt(fmt), group, _ptr(codes), _ptr(scale),
                            _ptr(zero), _stream(stream)), "wq_quantize")


def wq_gemv(x, codes, scale, zero, fmt, N, K, y, stream=None) -> None:
    _check(_lib.wq_gemv(_ptr(x), _ptr(codes), _ptr(scale), _ptr(zero), _fmt(fmt), N, K,
                        _ptr(y), _stream(stream)), "wq_gemv")


def wq_gemm(X, M, codes, scale, zero, fmt, N, K, Y, stream=None) -> None:
    _check(_lib.wq_gemm(_ptr(X), M, _ptr(codes), _ptr(scale), _ptr(zero), _fmt(fmt), N, K,
                        _ptr(Y), _stream(stream)), "wq_gemm")


def wq_argmax_workspace_bytes() -> int:
    return _lib.wq_argmax_workspace_bytes()


def wq_gemv_argmax(x, codes, scale, zero, fmt, N, K, y, argmax, workspace, workspace_bytes,
                   stream=None) -> None:
    """y may be None; argmax is a device int32 tensor; workspace a zero-filled device buffer."""
    _check(_lib.wq_gemv_argmax(_ptr(x), _ptr(codes), _ptr(scale), _ptr(zero), _fmt(fmt), N, K,
                               _ptr(y), _ptr(argmax), _ptr(workspace), workspace_bytes,
                               _stream(stream)), "wq_gemv_argmax")


def wq_gemv_argmax_static(x, codes, scale, zero, fmt, N, K, y, argmax, stream=None) -> None:
    """wq_gemv_argmax using the library's own static scratch (no work space argument)."""
    _check(_lib.wq_gemv_argmax_static(_ptr(x), _ptr(codes), _ptr(scale), _ptr(zero), _fmt(fmt),
                                      N, K, _ptr(y), _ptr(argmax), _stream(stream)),
           "wq_gemv_argmax_static")


def wq_rescore_workspace_bytes(N, topk) -> int:
    return _lib.wq_rescore_workspace_bytes(N, topk)


def wq_gemv_rescore(x, codes, scale, zero, fmt, w16, N, K, topk, y, cand, cand_logits, token,
                    workspace, workspace_bytes, stream=None) -> None:
    """Head rescoring: y (fp16 [N]), cand (int32 [topk]), cand_logits (fp32 [topk]) and
    token (int32 [1]) are device tensors; w16 is the fp16 head [N, K]."""
    _check(_lib.wq_gemv_rescore(_ptr(x), _ptr(codes), _ptr(scale), _ptr(zero), _fmt(fmt),
                                _ptr(w16), N, K, topk, _ptr(y), _ptr(cand), _ptr(cand_logits),
                                _ptr(token), _ptr(workspace), workspace_bytes, _stream(stream)),
           "wq_gemv_rescore")


def make_linear_set(entries) -> ctypes.Array:
    """Host descriptor array from (codes, scale, zero, x, y, N, K[, M]) tuples (M = 1 if omitted)."""
    arr = (wq_linear_desc * len(entries))()
    for i, e in enumerate(entries):
        c, s, z, x, y, N, K = e[:7]
        M = e[7] if len(e) > 7 else 1
        arr[i] = wq_linear_desc(_ptr(c), _ptr(s), _ptr(z), _ptr(x), _ptr(y), N, K, M)
    return arr


def wq_linear_set(descs, count, fmt, stream=None) -> None:
    _check(_lib.wq_linear_set(descs, count, _fmt(fmt), _stream(stream)), "wq_linear_set")


def wq_status_str(status: int) -> str:
    return _lib.wq_status_str(status).decode()


def wq_last_cuda_error() -> int:
    return _lib.wq_last_cuda_error()


def wq_device_errors(clear: bool = True, stream=None) -> int:
    """Device error flags (WQ_DEVERR_*) since the last clear; synchronises the stream."""
    f = ctypes.c_uint(0)
    _check(_lib.wq_device_errors(ctypes.byref(f), int(clear), _stream(stream)), "wq_device_errors")
    return f.value


WQ_DEVERR_TIMEOUT = 1


def wq_debug_arm_timeout(polls: int) -> None:
    """Failure-detection test hook: the next streaming-kernel launch on this thread has one
    unfilled ring slot and waits of at most `polls` polls (0 disarms)."""
    _check(_lib.wq_debug_arm_timeout(int(polls)), "wq_debug_arm_timeout")


# ---- allocation helpers (torch owns the memory) ------------------------------------

def alloc_packed(N: int, K: int, fmt, device="cuda"):
    """Empty (codes, scale, zero) tensors for an [N, K] weight; zero is None for ternary.
    scale holds fp16 bits (int16); zero too, except for int4h, whose zero is the index bytes
    (uint8 [N * K / 32]) and whose scale is the row pairs (int16 [2 N])."""
    f = _fmt(fmt)
    nbytes = wq_codes_bytes(f, N, K)
    if nbytes == 0:
        raise WQError(WQ_ERR_SHAPE, "alloc_packed")
    codes = torch.empty(nbytes, dtype=torch.uint8, device=device)
    scale = torch.empty(wq_scale_bytes(f, N, K) // 2, dtype=torch.int16, device=device)
    zb = wq_zero_bytes(f, N, K)
    if f == WQ_TERNARY:
        zero = None
    elif f == WQ_INT4H:
        zero = torch.empty(zb, dtype=torch.uint8, device=device)
    else:
        zero = torch.empty(zb // 2, dtype=torch.int16, device=device)
    return codes, scale, zero
