"""Head rescoring (wq_gemv_rescore) against the oracle.

The candidates are the top-k of the quantised head's own logits y (identical to wq_gemv's),
so they are compared exactly, ties included, with the oracle's top-k of that y; the
recomputed logits are compared with the oracle's float64 product of x and the fp16 rows
(|l - l_ref| <= 2e-3 sum|x w16|); the token must be the oracle's pick over the GPU's own
recomputed logits (largest, then lowest row).
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth
from oracle import wq_oracle as O

from gpu_util import assert_within_tol, quantize_gpu, wq

pytestmark = pytest.mark.gpu


def _run(W, x, fmt, topk):
    N, K = W.shape
    c, s, z = quantize_gpu(W.cuda(), fmt)
    w16 = W.half().cuda()  # the fp16 copy of the head
    xd = x.cuda()
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    cand = torch.full((topk,), -1, dtype=torch.int32, device="cuda")
    cl = torch.full((topk,), float("nan"), dtype=torch.float32, device="cuda")
    tok = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    wsb = wq().wq_rescore_workspace_bytes(N, topk)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    wq().wq_gemv_rescore(xd, c, s, z, fmt, w16, N, K, topk, y, cand, cl, tok, ws, wsb)
    torch.cuda.synchronize()
    y1 = torch.empty_like(y)
    wq().wq_gemv(xd, c, s, z, fmt, N, K, y1)
    torch.cuda.synchronize()
    assert torch.equal(y, y1), "y differs from wq_gemv"
    k = min(topk, N)
    got = cand.cpu().numpy()[:k].astype(np.int64)
    assert got.tolist() == O.topk_rows(y.cpu().numpy(), topk).tolist(), "candidates"
    ref, bound = O.rescore(x.numpy(), w16.cpu().numpy()[got])
    lg = cl.cpu().numpy()[:k].astype(np.float64)
    assert_within_tol(lg, ref, bound, f"rescore {fmt} {N}x{K} k={topk}")
    assert int(tok.item()) == O.pick_token(got, lg), "token"
    return got, lg, int(tok.item())


@pytest.mark.parametrize("fmt", ["int4", "int2", "ternary"])
@pytest.mark.parametrize("N,K", [(1, 128), (333, 896), (5000, 1024)])
@pytest.mark.parametrize("topk", [1, 8, 64])
def test_rescore_matches_oracle(fmt, N, K, topk):
    W = synth.weights(N, K, 0.02, seed=60 + N + topk)
    x = synth.activations(1, K, seed=61 + N)[0]
    _run(W, x, fmt, topk)


@pytest.mark.parametrize("topk", [8, 64])
def test_rescore_lm_head_int4(topk):
    N, K = 151936, 896
    W = synth.weights(N, K, 0.02, seed=62, device="cuda").cpu()
    x = synth.activations(1, K, seed=63)[0]
    _run(W, x, "int4", topk)


def test_rescore_ties_go_to_the_lower_row():
    N, K = 2100, 256   # two chunks of 2048 logits: the tied rows sit in both
    W = synth.weights(N, K, 0.02, seed=64)
    x = synth.activations(1, K, seed=65)[0]
    best = 3 * W[7].abs() * torch.sign(x.float())      # a row with a large positive logit
    for r in (2099, 7, 2050, 300):
        W[r] = best
    got, lg, tok = _run(W, x, "int4", 8)
    assert got[:4].tolist() == [7, 300, 2050, 2099]
    assert tok == 7
