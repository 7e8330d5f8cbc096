"""Parity of the fallback products that the common workloads never reach.

- Scales and zeros at a 2-byte (not 16-byte) offset: the streaming kernel needs 16-byte
  aligned metadata for its bulk copies, so batch-1 int4 / int2 products run on the
  row-per-lane kernel instead (wq.h allows 2-byte aligned scale and zero).
- K too long to stage the activations in shared memory (K = 131072): neither the streaming
  nor the row kernel takes it, and the generic set kernel does.
Both against the oracle, element by element within the product bound.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth

from gpu_util import assert_within_tol, f16_np, oracle_rows, quantize_gpu, wq

pytestmark = pytest.mark.gpu


def _offset_copy(t: torch.Tensor) -> torch.Tensor:
    """The same fp16 values in a buffer that starts 2 bytes past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
    v = buf[1:1 + t.numel()]
    v.copy_(t.reshape(-1))
    assert v.data_ptr() % 16 == 2
    return v


@pytest.mark.parametrize("fmt", ["int4", "int2"])
@pytest.mark.parametrize("N,K", [(300, 896), (64, 4864), (1, 128)])
def test_metadata_at_2_byte_offset(fmt, N, K):
    W = synth.weights(N, K, 0.02, seed=90 + N)
    x = synth.activations(1, K, seed=91 + K)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    s2, z2 = _offset_copy(scale), _offset_copy(zero)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    y_ref16 = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x.cuda(), codes, s2, z2, fmt, N, K, y)
    wq().wq_gemv(x.cuda(), codes, scale, zero, fmt, N, K, y_ref16)
    _, y_ref, bound = oracle_rows(W.numpy(), x.numpy(), fmt)
    assert_within_tol(f16_np(y), y_ref, bound, f"offset metadata {fmt} {N}x{K}")
    assert_within_tol(f16_np(y_ref16), y_ref, bound, f"aligned metadata {fmt} {N}x{K}")
    # a set of such matrices takes the same fallback
    ent = [(codes, s2, z2, x.cuda(), torch.empty(N, dtype=torch.float16, device="cuda"), N, K)] * 1
    wq().wq_linear_set(wq().make_linear_set(ent), 1, fmt)
    torch.cuda.synchronize()
    assert torch.equal(ent[0][4], y)


@pytest.mark.parametrize("fmt", ["int4", "int2"])
def test_activations_too_long_to_stage(fmt):
    N, K = 40, 131072
    W = synth.weights(N, K, 0.02, seed=95)
    x = synth.activations(1, K, seed=96)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x.cuda(), codes, scale, zero, fmt, N, K, y)
    _, y_ref, bound = oracle_rows(W.numpy(), x.numpy(), fmt)
    assert_within_tol(f16_np(y), y_ref, bound, f"long K {fmt}")
