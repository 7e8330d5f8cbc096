"""int3 g128 (3-bit codes in each row's little-endian bit stream) against the oracle:
quantiser bit-exact (codes, scales, zeros), products within 2e-3 * sum|x w_hat| for
batch 1 and several M, sets equal to single calls bit for bit, the exact special cases
(one-hot activations pick a column of w_hat rounded once; codes at the zero point give 0),
and sampled rows of the full lm_head."""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth
from oracle import wq_oracle as O

from gpu_util import (assert_bitexact, assert_within_tol, f16_np, oracle_rows, quantize_gpu,
                      rows_np, wq)
from test_gpu_parity import _crafted_weights

pytestmark = pytest.mark.gpu

SHAPES = [(1, 128), (7, 256), (333, 896), (45, 4864), (200, 1152)]


@pytest.mark.parametrize("N,K", SHAPES)
def test_int3_quantize_bitexact(N, K):
    W = _crafted_weights(N, K, seed=1300 + N)
    c, s, z = quantize_gpu(W.cuda(), "int3")
    p, sb, zb = O.quantize(W.numpy(), "int3")
    assert_bitexact(rows_np(c, s, z, "int3", N, K), (p, sb, zb), f"int3 quantise {N}x{K}")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 17])
@pytest.mark.parametrize("N,K", SHAPES)
def test_int3_product_matches_oracle(M, N, K):
    W = _crafted_weights(N, K, seed=1400 + N)
    X = synth.activations(M, K, seed=1500 + M)
    c, s, z = quantize_gpu(W.cuda(), "int3")
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    wq().wq_gemm(X.cuda(), M, c, s, z, "int3", N, K, Y)
    torch.cuda.synchronize()
    _, y_ref, bound = oracle_rows(W.numpy(), X.numpy(), "int3")
    assert_within_tol(f16_np(Y), y_ref, bound, f"int3 M={M} {N}x{K}")
    if M == 1:
        y1 = torch.empty(N, dtype=torch.float16, device="cuda")
        wq().wq_gemv(X[0].cuda(), c, s, z, "int3", N, K, y1)
        assert torch.equal(y1, Y[0])


@pytest.mark.parametrize("M", [1, 3])
def test_int3_set_equals_single_calls(M):
    ent, singles = [], []
    for i, (N, K) in enumerate(SHAPES):
        W = synth.weights(N, K, 0.02, seed=1600 + i)
        X = synth.activations(M, K, seed=1700 + i).cuda()
        c, s, z = quantize_gpu(W.cuda(), "int3")
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        Ys = torch.empty(M, N, dtype=torch.float16, device="cuda")
        wq().wq_gemm(X, M, c, s, z, "int3", N, K, Ys)
        ent.append((c, s, z, X, Y, N, K, M))
        singles.append(Ys)
    wq().wq_linear_set(wq().make_linear_set(ent), len(ent), "int3")
    torch.cuda.synchronize()
    for (c, s, z, X, Y, N, K, _), Ys in zip(ent, singles):
        assert torch.equal(Y, Ys), (M, N, K)


def test_int3_special_cases():
    N, K = 40, 512
    W = synth.weights(N, K, 0.02, seed=1800)
    c, s, z = quantize_gpu(W.cuda(), "int3")
    p, sb, zb = O.quantize(W.numpy(), "int3")
    w_hat = O.dequant_int(p, sb, zb, 3, K)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    for k in (0, 10, 21, 31, 127, 128, 330, K - 1):   # codes 10 and 21 straddle two words
        x = torch.zeros(K, dtype=torch.float16)
        x[k] = 1.0
        wq().wq_gemv(x.cuda(), c, s, z, "int3", N, K, y)
        assert np.array_equal(f16_np(y), O.f16_round(w_hat[:, k])), k
    zq = np.repeat(O.f16_from_bits(zb), 128, axis=1).astype(np.int64)
    cz = torch.from_numpy(O.pack_int(zq, 3).view(np.uint8).reshape(-1)).cuda()
    wq().wq_gemv(synth.activations(1, K, seed=1801)[0].cuda(), cz, s, z, "int3", N, K, y)
    assert torch.all(y == 0)


def test_int3_lm_head_sampled():
    N, K = 151936, 896
    W = synth.weights(N, K, 0.02, seed=1900, device="cuda")
    c, s, z = quantize_gpu(W, "int3")
    x = synth.activations(1, K, seed=1901, device="cuda")[0]
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x, c, s, z, "int3", N, K, y)
    torch.cuda.synchronize()
    rows = np.array(sorted(set(np.random.default_rng(3).choice(N, 256, replace=False).tolist()) | {0, N - 1}))
    Wr = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    packed, y_ref, bound = oracle_rows(Wr, x.cpu().numpy(), "int3")
    assert_bitexact(rows_np(c, s, z, "int3", N, K, rows), packed, "int3 lm_head quantise")
    assert_within_tol(f16_np(y)[rows], y_ref, bound, "int3 lm_head")
