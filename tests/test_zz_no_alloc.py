"""wq_gemv_argmax_static: the fused product + greedy pick for callers that cannot allocate.

Engines that own all device memory through their own pool, or decode loops where an
allocation is not allowed, cannot hand libwq a work space; this entry point uses a static
array inside the library instead. It must give the same outputs and the same picked row as
wq_gemv_argmax with a caller work space, call after call (the static array is reused and
keeps the previous call's contents). This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth

from gpu_util import f16_np, quantize_gpu, wq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["int4", "int2"])
def test_static_scratch_matches_work_space_version(fmt):
    lib = wq()
    N, K = 151936, 896
    W = synth.weights(N, K, 0.02, seed=77)
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    ws = torch.zeros(lib.wq_argmax_workspace_bytes(), dtype=torch.uint8, device="cuda")
    am_ref = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    y_ref = torch.empty(N, dtype=torch.float16, device="cuda")
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    for call in range(2):  # two calls in a row: the static array is reused as the first left it
        x = synth.activations(1, K, seed=78 + call)[0].cuda()
        lib.wq_gemv_argmax(x, codes, scale, zero, fmt, N, K, y_ref, am_ref, ws, ws.numel())
        am.fill_(-1)
        y.fill_(float("nan"))
        # straight through the C ABI, as a caller without Python helpers would
        st = lib._lib.wq_gemv_argmax_static(x.data_ptr(), codes.data_ptr(), scale.data_ptr(),
                                            zero.data_ptr(), lib.FMT[fmt], N, K, y.data_ptr(),
                                            am.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == lib.WQ_OK, lib.wq_status_str(st)
        torch.cuda.synchronize()
        assert am.item() == am_ref.item(), call
        assert np.array_equal(f16_np(y), f16_np(y_ref)), call  # same kernel: identical outputs


def test_static_scratch_rejects_before_any_launch():
    lib = wq()
    x = torch.zeros(256, dtype=torch.float16, device="cuda")
    am = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = lib._lib.wq_gemv_argmax_static(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                        lib.WQ_TERNARY, 4, 256, None, am.data_ptr(), None)
    assert st == lib.WQ_ERR_ARG
    st = lib._lib.wq_gemv_argmax_static(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                        lib.WQ_INT4, 4, 100, None, am.data_ptr(), None)
    assert st == lib.WQ_ERR_SHAPE
    assert lib.wq_argmax_workspace_bytes() <= lib.WQ_ARGMAX_STATIC_SCRATCH_BYTES
