"""Fused product + greedy pick (wq_gemv_argmax) against the unfused product and the oracle.

The pick is made on the fp16 outputs (ties to the lowest row), so it must equal the argmax
of the y that wq_gemv writes; against the float64 oracle, whose outputs differ within the
product tolerance, the picked row must be a valid maximum within that tolerance.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth
from oracle import wq_oracle as O

from gpu_util import TOL, f16_np, oracle_rows, quantize_gpu, wq

pytestmark = pytest.mark.gpu


def _workspace():
    nb = wq().wq_argmax_workspace_bytes()
    assert nb > 16
    return torch.zeros(nb, dtype=torch.uint8, device="cuda"), nb


def _first_max(v):
    """Index of the largest value, the lowest one among equals."""
    return int(np.flatnonzero(v == v.max())[0])


@pytest.mark.parametrize("fmt", ["int4", "int2"])
@pytest.mark.parametrize("N,K", [(1, 128), (333, 896), (1000, 1152), (4096, 4864), (151936, 896)])
def test_argmax_matches_unfused_and_oracle(fmt, N, K):
    W = synth.weights(N, K, 0.02, seed=40 + N % 97 + K)
    x = synth.activations(1, K, seed=41 + K)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    xd = x.cuda()
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    y2 = torch.empty(N, dtype=torch.float16, device="cuda")
    am = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    ws, nb = _workspace()
    wq().wq_gemv(xd, codes, scale, zero, fmt, N, K, y)
    wq().wq_gemv_argmax(xd, codes, scale, zero, fmt, N, K, y2, am[0:], ws, nb)
    wq().wq_gemv_argmax(xd, codes, scale, zero, fmt, N, K, None, am[1:], ws, nb)  # y not stored
    torch.cuda.synchronize()
    yg = f16_np(y)
    assert np.array_equal(f16_np(y2), yg)                 # same product, bit for bit
    i0, i1 = am.cpu().tolist()
    assert i0 == i1 == _first_max(yg)
    assert ws[:4].cpu().tolist() == [0, 0, 0, 0]          # ticket counter back to zero
    # the oracle's largest output lies among the GPU's 64 largest (its outputs are within the
    # tolerance, far below the spread of the top values), so those rows are enough
    rows = np.unique(np.r_[i0, np.argsort(yg, kind="stable")[-64:]])
    _, y_ref, bound = oracle_rows(W.numpy()[rows], x.numpy(), fmt)
    top = np.max(y_ref)
    j = int(np.flatnonzero(rows == i0)[0])
    assert y_ref[j] >= top - 2 * TOL * np.max(bound)      # a maximum within the tolerance


@pytest.mark.parametrize("fmt", ["int4", "int2"])
def test_argmax_ties_go_to_the_lowest_row(fmt):
    N, K = 2000, 896
    W = synth.weights(N, K, 0.02, seed=7)
    x = synth.activations(1, K, seed=8)[0]
    hot = torch.sign(x.float()) * 0.5                     # rows aligned with x: the largest outputs
    for r in (1500, 37, 999):
        W[r] = hot
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ws, nb = _workspace()
    for _ in range(3):                                    # the work space is reused as left
        am.fill_(-1)
        wq().wq_gemv_argmax(x.cuda(), codes, scale, zero, fmt, N, K, None, am, ws, nb)
        torch.cuda.synchronize()
        assert am.item() == 37


def test_argmax_rejects_bad_arguments():
    N, K = 64, 256
    W = synth.weights(N, K, 0.02, seed=9)
    codes, scale, zero = quantize_gpu(W.cuda(), "int4")
    x = torch.zeros(K, dtype=torch.float16, device="cuda")
    am = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws, nb = _workspace()
    with pytest.raises(wq().WQError):                     # work space too small
        wq().wq_gemv_argmax(x, codes, scale, zero, "int4", N, K, None, am, ws, 8)
    c3, s3, _ = quantize_gpu(W.cuda(), "ternary")
    with pytest.raises(wq().WQError):                     # ternary is not served
        wq().wq_gemv_argmax(x, c3, s3, None, "ternary", N, K, None, am, ws, nb)


@pytest.mark.parametrize("fmt", ["int4", "int2", "int4h"])
def test_argmax_all_outputs_minus_infinity(fmt):
    """Finite inputs whose products overflow fp16 to -inf in every row: the pick is still a
    valid row, the lowest one (all values tie)."""
    lib = wq()
    N, K = 300, 128
    codes, scale, zero = lib.alloc_packed(N, K, fmt)
    codes.zero_()  # every code 0
    if fmt == "int4h":
        # w_hat = d a q - dm b: q = 0, dm = 1000, b = 15 -> -15000 per weight
        pair = torch.tensor([0x3C00, 0x63D0], dtype=torch.int32).to(torch.int16).repeat(N)
        scale.copy_(pair.cuda())
        zero.fill_(0xF1)  # index byte: a = 1, b = 15
    else:
        scale.fill_(0x63D0)  # fp16 1000
        zero.fill_(0x4B80 if fmt == "int4" else 0x4200)  # fp16 15 (int4) / 3 (int2): w_hat < 0
    x = torch.full((K,), 60000.0, dtype=torch.float16, device="cuda")
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ws, nb = _workspace()
    lib.wq_gemv_argmax(x, codes, scale, zero, fmt, N, K, y, am, ws, nb)
    torch.cuda.synchronize()
    assert torch.all(torch.isinf(y.float()) & (y.float() < 0)), "every output overflows to -inf"
    assert int(am.item()) == 0
