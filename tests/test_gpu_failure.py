"""Failure detection: a bounded wait inside the streaming kernel runs out, on purpose.

wq_debug_arm_timeout makes the next streaming-kernel launch leave one ring slot of CTA 0's
warp 0 unfilled, with every mbarrier wait bounded by a few thousand polls. The wait on that
slot gives up; the kernel stops computing, waits (bounded) for its other copies, sets
WQ_DEVERR_TIMEOUT and returns. No GPU fault, trap or hang is involved: the call returns, the
context stays usable, and the next call on the same stream is correct.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth

from gpu_util import assert_within_tol, f16_np, oracle_rows, quantize_gpu, wq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["int4", "int2"])
def test_bounded_wait_gives_up_reports_and_recovers(fmt):
    # enough rows that CTA 0's warp 0 has units of work (its first slot is the one left empty)
    N, K = 32768, 896
    W = synth.weights(N, K, 0.02, seed=77)
    x = synth.activations(1, K, seed=78)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    xd = x.cuda()
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    lib = wq()
    lib.wq_device_errors(clear=True)                     # start from clean flags
    lib.wq_debug_arm_timeout(2000)
    lib.wq_gemv(xd, codes, scale, zero, fmt, N, K, y)   # returns: the kernel gives up, not hangs
    flags = lib.wq_device_errors(clear=True)            # synchronises the stream
    assert flags & lib.WQ_DEVERR_TIMEOUT
    # the hook was consumed by that launch: the next call runs normally and is correct
    y.fill_(float("nan"))
    lib.wq_gemv(xd, codes, scale, zero, fmt, N, K, y)
    assert lib.wq_device_errors(clear=True) == 0
    rows = np.r_[np.arange(256), np.random.default_rng(3).choice(N, 256, replace=False)]
    _, y_ref, bound = oracle_rows(W.numpy()[rows], x.numpy(), fmt)
    assert_within_tol(f16_np(y)[rows], y_ref, bound, f"after timeout {fmt}")


def test_disarmed_hook_changes_nothing():
    N, K = 2048, 896
    W = synth.weights(N, K, 0.02, seed=79)
    x = synth.activations(1, K, seed=80)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), "int4")
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    lib = wq()
    lib.wq_device_errors(clear=True)
    lib.wq_debug_arm_timeout(2000)
    lib.wq_debug_arm_timeout(0)                          # disarmed again before any launch
    lib.wq_gemv(x.cuda(), codes, scale, zero, "int4", N, K, y)
    assert lib.wq_device_errors(clear=True) == 0
    _, y_ref, bound = oracle_rows(W.numpy(), x.numpy(), "int4")
    assert_within_tol(f16_np(y), y_ref, bound, "disarmed")
