"""The C-ABI library loads and exports every entry point wq.h declares (no GPU needed).

Only host-side logic is exercised: size queries and the argument checks that reject a
call before anything touches CUDA.
"""
import ctypes
import os
import re

import pytest

from bit_weight_quantized_unpack_b200 import build as wq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(wq_build.build())


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(wq_\w+)\s*\(", src, re.M))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"wq_quantize", "wq_gemv", "wq_gemm", "wq_linear_set", "wq_codes_bytes",
            "wq_meta_count", "wq_status_str", "wq_last_cuda_error"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_sizes(lib):
    lib.wq_codes_bytes.restype = ctypes.c_size_t
    lib.wq_codes_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64]
    lib.wq_meta_count.restype = ctypes.c_size_t
    lib.wq_meta_count.argtypes = [ctypes.c_int64, ctypes.c_int64]
    assert lib.wq_codes_bytes(0, 151936, 896) == 151936 * 448
    assert lib.wq_codes_bytes(1, 151936, 896) == 151936 * 224
    assert lib.wq_codes_bytes(2, 151936, 896) == 151936 * 182
    assert lib.wq_codes_bytes(3, 151936, 896) == 151936 * 336     # int3: 3 bits per code
    assert lib.wq_meta_count(151936, 896) == 151936 * 7
    # stored bits per weight of the layout: 4.25, 2.25, 1.75, 3.25
    for fmt, bpw in ((0, 4.25), (1, 2.25), (2, 1.75), (3, 3.25)):
        meta_arrays = 1 if fmt == 2 else 2          # scale (+ zero), fp16 each
        tot = lib.wq_codes_bytes(fmt, 64, 1024) + 2 * meta_arrays * lib.wq_meta_count(64, 1024)
        assert tot * 8 / (64 * 1024) == bpw
    assert lib.wq_codes_bytes(0, 4, 100) == 0      # K not a multiple of 128
    assert lib.wq_codes_bytes(5, 4, 128) == 0      # unknown format
    assert lib.wq_codes_bytes(0, 0, 128) == 0
    # int4h: int4 codes + one index byte per 32 weights + one fp16 pair per row; the stored
    # bits per weight are 4 + 8/32 + 32/K (the Whetstone README format table's 4.28 is the
    # whole-model figure, pinned in the oracle tests)
    for f in ("wq_scale_bytes", "wq_zero_bytes"):
        getattr(lib, f).restype = ctypes.c_size_t
        getattr(lib, f).argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64]
    N, K = 151936, 896
    assert lib.wq_codes_bytes(4, N, K) == N * K // 2
    assert lib.wq_scale_bytes(4, N, K) == 4 * N
    assert lib.wq_zero_bytes(4, N, K) == N * K // 32
    tot = lib.wq_codes_bytes(4, N, K) + lib.wq_scale_bytes(4, N, K) + lib.wq_zero_bytes(4, N, K)
    assert tot * 8 / (N * K) == pytest.approx(4 + 8 / 32 + 32 / K, rel=1e-12)
    for fmt in (0, 1, 3):
        assert lib.wq_scale_bytes(fmt, N, K) == lib.wq_zero_bytes(fmt, N, K) == 2 * N * 7
    assert lib.wq_scale_bytes(2, N, K) == 2 * N * 7 and lib.wq_zero_bytes(2, N, K) == 0
    assert lib.wq_scale_bytes(5, N, K) == 0 and lib.wq_zero_bytes(4, N, 100) == 0


def test_argument_checks_reject_before_any_launch(lib):
    from bit_weight_quantized_unpack_b200 import wq
    P = 1 << 20   # a 16-byte aligned fake address: never dereferenced on a rejected call
    S = None      # stream
    # null pointers, bad format, bad group
    assert wq._lib.wq_gemv(None, P, P, P, 0, 8, 128, P, S) == wq.WQ_ERR_ARG
    assert wq._lib.wq_gemv(P, P, P, None, 0, 8, 128, P, S) == wq.WQ_ERR_ARG      # int4 needs zero
    assert wq._lib.wq_gemv(P, P, P, P, 2, 8, 128, P, S) == wq.WQ_ERR_ARG         # ternary: no zero
    assert wq._lib.wq_gemv(P, P, P, P, 7, 8, 128, P, S) == wq.WQ_ERR_ARG
    assert wq._lib.wq_quantize(P, 8, 128, 0, 64, P, P, P, S) == wq.WQ_ERR_ARG
    # shapes
    assert wq._lib.wq_gemv(P, P, P, P, 0, 8, 100, P, S) == wq.WQ_ERR_SHAPE
    assert wq._lib.wq_gemv(P, P, P, P, 0, 0, 128, P, S) == wq.WQ_ERR_SHAPE
    assert wq._lib.wq_gemv(P, P, P, P, 0, 8, 0, P, S) == wq.WQ_ERR_SHAPE
    assert wq._lib.wq_gemm(P, 0, P, P, P, 0, 8, 128, P, S) == wq.WQ_ERR_SHAPE
    assert wq._lib.wq_gemm(P, 2049, P, P, P, 0, 8, 128, P, S) == wq.WQ_ERR_SHAPE
    # alignment
    assert wq._lib.wq_gemv(P + 8, P, P, P, 0, 8, 128, P, S) == wq.WQ_ERR_ALIGN
    assert wq._lib.wq_gemv(P, P + 4, P, P, 0, 8, 128, P, S) == wq.WQ_ERR_ALIGN
    assert wq._lib.wq_gemv(P, P, P + 1, P, 0, 8, 128, P, S) == wq.WQ_ERR_ALIGN
    assert wq._lib.wq_quantize(P + 4, 8, 128, 0, 128, P, P, P, S) == wq.WQ_ERR_ALIGN
    # int4h: group 32, row pairs 4-byte and index bytes 16-byte aligned
    assert wq._lib.wq_quantize(P, 8, 128, 4, 128, P, P, P, S) == wq.WQ_ERR_ARG
    assert wq._lib.wq_gemv(P, P, P + 2, P, 4, 8, 128, P, S) == wq.WQ_ERR_ALIGN
    assert wq._lib.wq_gemv(P, P, P, P + 4, 4, 8, 128, P, S) == wq.WQ_ERR_ALIGN
    assert wq._lib.wq_gemv(P, P, P, None, 4, 8, 128, P, S) == wq.WQ_ERR_ARG
    # linear set: count range, and a bad entry anywhere rejects the whole call
    good = (P, P, P, P, P, 8, 128)
    arr = wq.make_linear_set([good, (P, P, P, P, P, 8, 130)])
    assert wq._lib.wq_linear_set(arr, 2, 0, S) == wq.WQ_ERR_SHAPE
    assert wq._lib.wq_linear_set(arr, 0, 0, S) == wq.WQ_ERR_ARG
    assert wq._lib.wq_linear_set(arr, 257, 0, S) == wq.WQ_ERR_ARG
    assert wq._lib.wq_linear_set(None, 1, 0, S) == wq.WQ_ERR_ARG
    assert wq.wq_status_str(wq.WQ_ERR_ALIGN).startswith("WQ_ERR_ALIGN")


def test_rescore_sizes_and_argument_checks(lib):
    from bit_weight_quantized_unpack_b200 import wq
    # one 8-byte key per candidate and 2048-logit chunk
    assert wq.wq_rescore_workspace_bytes(151936, 8) == 75 * 8 * 8
    assert wq.wq_rescore_workspace_bytes(1, 1) == 8
    assert wq.wq_rescore_workspace_bytes(524288, 64) == 256 * 64 * 8
    assert wq.wq_rescore_workspace_bytes(524289, 8) == 0
    assert wq.wq_rescore_workspace_bytes(100, 0) == 0
    assert wq.wq_rescore_workspace_bytes(100, wq.WQ_RESCORE_MAX_TOPK + 1) == 0
    P = 1 << 20   # a 16-byte aligned fake address: never dereferenced on a rejected call
    ws = 1 << 16
    f = wq._lib.wq_gemv_rescore
    assert f(P, P, P, P, 0, None, 1000, 128, 8, P, P, P, P, P, ws, None) == wq.WQ_ERR_ARG   # no fp16 head
    assert f(P, P, P, P, 0, P, 1000, 128, 0, P, P, P, P, P, ws, None) == wq.WQ_ERR_ARG      # topk 0
    assert f(P, P, P, P, 0, P, 1000, 128, 65, P, P, P, P, P, ws, None) == wq.WQ_ERR_ARG     # topk > 64
    assert f(P, P, P, P, 0, P, 524289, 128, 8, P, P, P, P, P, ws, None) == wq.WQ_ERR_SHAPE  # too many rows
    assert f(P, P, P, P, 0, P, 1000, 100, 8, P, P, P, P, P, ws, None) == wq.WQ_ERR_SHAPE    # K % 128
    assert f(P, P, P, P, 0, P, 1000, 128, 8, P, P, P, P, P, 8, None) == wq.WQ_ERR_ARG       # small work space
    assert f(P, P, P, P, 0, P + 8, 1000, 128, 8, P, P, P, P, P, ws, None) == wq.WQ_ERR_ALIGN
    assert f(P, P, P, P, 0, P, 1000, 128, 8, P, P, P, P, P + 4, ws, None) == wq.WQ_ERR_ALIGN
