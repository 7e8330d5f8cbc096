"""Parity of the skinny-batch int4 GEMM (M = 2..32 tokens, warp-level MMAs fed from registers)
with the oracle, through wq_gemm / wq_linear_set.

Covers every token-block count (M up to 8, 16 and 32) and the M at their edges, weight
counts that are not multiples of the 16-row slab or the 128-row unit, K that fits one
activation chunk and K that needs several, the degenerate rows of the quantiser, a set of
matrices of different K (bit-identical to per-matrix calls), and the exact special cases
(one-hot activations pick a column of w_hat rounded once to fp16; codes equal to the zero
point give exact zeros).
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth
from oracle import wq_oracle as O

from gpu_util import assert_within_tol, f16_np, oracle_rows, quantize_gpu, wq
from test_gpu_parity import _crafted_weights

pytestmark = pytest.mark.gpu

MS = [2, 3, 4, 5, 7, 8, 9, 15, 16, 17, 24, 31, 32]
SHAPES = [(1, 128), (7, 256), (129, 896), (300, 1024), (333, 4864), (40, 7168)]


@pytest.mark.parametrize("M", MS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_skinny_gemm_matches_oracle(M, N, K):
    W = _crafted_weights(N, K, seed=700 + N)
    X = synth.activations(M, K, seed=800 + M)
    c, s, z = quantize_gpu(W.cuda(), "int4")
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    wq().wq_gemm(X.cuda(), M, c, s, z, "int4", N, K, Y)
    torch.cuda.synchronize()
    _, y_ref, bound = oracle_rows(W.numpy(), X.numpy(), "int4")
    assert_within_tol(f16_np(Y), y_ref, bound, f"skinny M={M} {N}x{K}")


@pytest.mark.parametrize("M", [2, 5, 16, 32])
def test_skinny_set_equals_single_calls(M):
    shapes = [(896, 896), (128, 896), (333, 1152), (40, 4864), (513, 256), (256, 128), (1000, 3584)]
    ent, singles = [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, 0.02, seed=900 + i)
        X = synth.activations(M, K, seed=950 + i).cuda()
        c, s, z = quantize_gpu(W.cuda(), "int4")
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        Ys = torch.empty(M, N, dtype=torch.float16, device="cuda")
        wq().wq_gemm(X, M, c, s, z, "int4", N, K, Ys)
        ent.append((c, s, z, X, Y, N, K, M))
        singles.append(Ys)
    wq().wq_linear_set(wq().make_linear_set(ent), len(ent), "int4")
    torch.cuda.synchronize()
    for (c, s, z, X, Y, N, K, _), Ys in zip(ent, singles):
        assert torch.equal(Y, Ys), (M, N, K)


@pytest.mark.parametrize("M", [2, 5, 12, 32])
def test_skinny_special_cases(M):
    N, K = 77, 1024
    W = synth.weights(N, K, 0.02, seed=11)
    codes, scale, zero = quantize_gpu(W.cuda(), "int4")
    p, s, z = O.quantize(W.numpy(), "int4")
    w_hat = O.dequant_int(p, s, z, 4, K)
    # token m of X is the one-hot vector e_{k_m}: row m of Y is column k_m of w_hat, rounded once
    ks = [(37 * m + 5) % K for m in range(M)]
    X = torch.zeros(M, K, dtype=torch.float16)
    for m, k in enumerate(ks):
        X[m, k] = 1.0
    Y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    wq().wq_gemm(X.cuda(), M, codes, scale, zero, "int4", N, K, Y)
    got = f16_np(Y)
    for m, k in enumerate(ks):
        assert np.array_equal(got[m], O.f16_round(w_hat[:, k])), (m, k)
    # codes equal to their group's zero point: w_hat = 0, so Y is exactly 0
    zq = np.repeat(O.f16_from_bits(z), 128, axis=1).astype(np.int64)
    cz = torch.from_numpy(O.pack_int(zq, 4).view(np.uint8).reshape(-1)).cuda()
    Xr = synth.activations(M, K, seed=12).cuda()
    wq().wq_gemm(Xr, M, cz, scale, zero, "int4", N, K, Y)
    assert torch.all(Y == 0)
