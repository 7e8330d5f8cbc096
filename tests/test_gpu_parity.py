"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Quantiser: codes, scales and zeros bit-exact. Products: |y_gpu - y_ref| <= 2e-3 * sum|x w_hat|
per element (y_ref and the bound from the oracle's own quantisation of the same W).
Small cases are checked element by element; the full-size workloads, in the launch
configuration the bench times, on sampled rows.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth, workloads
from oracle import wq_oracle as O

from gpu_util import (assert_bitexact, assert_within_tol, f16_np, oracle_rows, quantize_gpu,
                      rows_np, wq)

pytestmark = pytest.mark.gpu

FMTS = ("int4", "int2", "ternary")


def _crafted_weights(N, K, seed):
    """Seeded N(0, 0.02^2) weights plus rows that hit the degenerate and tie cases."""
    W = synth.weights(N, K, 0.02, seed)
    if N >= 6:
        W[0] = 0.0                                    # zero rows: s = 1, z = 0, codes 0
        W[1] = 0.3                                    # constant rows
        W[2] *= 8.0                                   # an outlier row
        j = torch.arange(K)
        W[3] = -1 + 0.125 * (j % 16)                  # exact ramp: codes 0..15
        W[4] = W[3] + 0.0625                          # every w / s is a tie x.5
        W[4, ::16] = -1.0                             # keep lo = -1, hi = 0.875 per group
        W[4, 15::16] = 0.875
        W[5, : K // 2] = -0.0                         # signed zeros
        W[5, K // 2:] = 0.0
    return W


SMALL = [(1, 128), (7, 256), (64, 896), (333, 896), (200, 1152), (45, 4864), (1000, 128)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SMALL)
def test_quantize_bitexact_small(fmt, N, K):
    W = _crafted_weights(N, K, seed=11 + N + K)
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    torch.cuda.synchronize()
    assert_bitexact(rows_np(codes, scale, zero, fmt, N, K), O.quantize(W.numpy(), fmt),
                    f"{fmt} {N}x{K}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SMALL)
def test_gemv_small(fmt, N, K):
    W = _crafted_weights(N, K, seed=21 + N + K)
    x = synth.activations(1, K, seed=31 + K)[0]
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x.cuda(), codes, scale, zero, fmt, N, K, y)
    _, y_ref, bound = oracle_rows(W.numpy(), x.numpy(), fmt)
    assert_within_tol(f16_np(y), y_ref, bound, f"gemv {fmt} {N}x{K}")


@pytest.mark.parametrize("fmt", FMTS)
def test_gemv_special_cases(fmt):
    N, K = 40, 512
    W = synth.weights(N, K, 0.02, seed=5)
    codes, scale, zero = quantize_gpu(W.cuda(), fmt)
    p, s, z = O.quantize(W.numpy(), fmt)
    w_hat = (O.dequant_ternary(p, s, K) if fmt == "ternary"
             else O.dequant_int(p, s, z, {"int4": 4, "int2": 2}[fmt], K))
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    # x = e_k picks column k of w_hat, rounded once to fp16
    for k in (0, 1, 127, 128, 300, K - 1):
        x = torch.zeros(K, dtype=torch.float16)
        x[k] = 1.0
        wq().wq_gemv(x.cuda(), codes, scale, zero, fmt, N, K, y)
        assert np.array_equal(f16_np(y), O.f16_round(w_hat[:, k])), k
    # a zero activation vector gives exactly 0
    wq().wq_gemv(torch.zeros(K, dtype=torch.float16, device="cuda"), codes, scale, zero, fmt, N, K, y)
    assert torch.all(y == 0)
    if fmt != "ternary":
        # all codes equal to their group's zero point -> w_hat = 0 -> y exactly 0
        zq = np.repeat(O.f16_from_bits(z), 128, axis=1).astype(np.int64)
        cz = torch.from_numpy(O.pack_int(zq, {"int4": 4, "int2": 2}[fmt]).view(np.uint8).reshape(-1))
        x = synth.activations(1, K, seed=6)[0].cuda()
        wq().wq_gemv(x, cz.cuda(), scale, zero, fmt, N, K, y)
        assert torch.all(y == 0)


def test_linear_set_small_matches_gemv_and_oracle():
    shapes = [(896, 896), (128, 896), (4864, 896), (896, 4864), (1, 128), (333, 1152),
              (77, 3584), (40, 18944), (513, 256)]
    for fmt in FMTS:
        ent, refs, outs, singles = [], [], [], []
        for i, (N, K) in enumerate(shapes):
            W = synth.weights(N, K, 0.02, seed=100 + i)
            x = synth.activations(1, K, seed=200 + i)[0]
            c, s, z = quantize_gpu(W.cuda(), fmt)
            xd = x.cuda()
            y = torch.full((N,), float("nan"), dtype=torch.float16, device="cuda")
            ys = torch.empty(N, dtype=torch.float16, device="cuda")
            wq().wq_gemv(xd, c, s, z, fmt, N, K, ys)
            ent.append((c, s, z, xd, y, N, K))
            outs.append(y)
            singles.append(ys)
            refs.append(oracle_rows(W.numpy(), x.numpy(), fmt)[1:])
        arr = wq().make_linear_set(ent)
        wq().wq_linear_set(arr, len(ent), fmt)
        torch.cuda.synchronize()
        for (y_ref, bound), y, ys, shp in zip(refs, outs, singles, shapes):
            assert torch.equal(y, ys), (fmt, shp)            # same kernel, same result
            assert_within_tol(f16_np(y), y_ref, bound, f"set {fmt} {shp}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [2, 5, 16, 37, 300])
def test_linear_set_batched_matches_gemm_and_oracle(fmt, M):
    """A set of M-row products (tensor-core path for int4 at M >= 16, over more matrices
    than one tensor-core launch takes) equals per-matrix wq_gemm and the oracle."""
    base = [(896, 896), (128, 896), (333, 1152), (40, 4864), (513, 256), (256, 128)]
    shapes = base * (15 if (fmt == "int4" and M == 16) else 1)  # 90 > 80 matrices per launch
    ent, checks = [], []
    for i, (N, K) in enumerate(shapes):
        W = synth.weights(N, K, 0.02, seed=300 + i)
        X = synth.activations(M, K, seed=400 + i)
        c, s, z = quantize_gpu(W.cuda(), fmt)
        Xd = X.cuda()
        Y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        Ys = torch.empty(M, N, dtype=torch.float16, device="cuda")
        wq().wq_gemm(Xd, M, c, s, z, fmt, N, K, Ys)
        ent.append((c, s, z, Xd, Y, N, K, M))
        ref = oracle_rows(W.numpy(), X.numpy(), fmt)[1:] if i < len(base) else None
        checks.append((Y, Ys, ref, (N, K)))
    wq().wq_linear_set(wq().make_linear_set(ent), len(ent), fmt)
    torch.cuda.synchronize()
    for Y, Ys, ref, shp in checks:
        assert torch.equal(Y, Ys), (fmt, M, shp)
        if ref is not None:
            assert_within_tol(f16_np(Y), ref[0], ref[1], f"set {fmt} M={M} {shp}")


def test_linear_set_rejects_mixed_m():
    c, s, z = quantize_gpu(synth.weights(128, 128, 0.02, 1).cuda(), "int4")
    x = torch.zeros(2, 128, dtype=torch.float16, device="cuda")
    y = torch.zeros(2, 128, dtype=torch.float16, device="cuda")
    arr = wq().make_linear_set([(c, s, z, x, y, 128, 128, 2), (c, s, z, x, y, 128, 128, 1)])
    with pytest.raises(wq().WQError):
        wq().wq_linear_set(arr, 2, "int4")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 17])
def test_gemm_small(fmt, M):
    N, K = 300, 1024
    W = synth.weights(N, K, 0.02, seed=40 + M)
    X = synth.activations(M, K, seed=50 + M)
    c, s, z = quantize_gpu(W.cuda(), fmt)
    Y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    wq().wq_gemm(X.cuda(), M, c, s, z, fmt, N, K, Y)
    _, y_ref, bound = oracle_rows(W.numpy(), X.numpy(), fmt)
    assert_within_tol(f16_np(Y), y_ref, bound, f"gemm {fmt} M={M}")
    if M == 1:
        y1 = torch.empty(N, dtype=torch.float16, device="cuda")
        wq().wq_gemv(X[0].cuda(), c, s, z, fmt, N, K, y1)
        assert torch.equal(y1, Y[0])


# ---- full-size workloads, sampled rows --------------------------------------------

def _sample_rows(N, k, seed, extra=()):
    g = np.random.default_rng(seed)
    r = set(g.choice(N, size=min(k, N), replace=False).tolist()) | {0, N - 1} | set(extra)
    return np.array(sorted(r))


def _check_set_sampled(widx, fmt="int4", rows_per_mat=48):
    wl = workloads.WORKLOADS[widx]
    mats = workloads.workload_mats(widx)
    ent, keep = [], []
    for i, m in enumerate(mats):
        W = synth.weights(m.N, m.K, wl["sigma"], synth.sub_seed(wl["seed"], i, 0), device="cuda")
        c, s, z = quantize_gpu(W, fmt)
        x = synth.activations(1, m.K, synth.sub_seed(wl["seed"], i, 1), device="cuda")[0]
        y = torch.empty(m.N, dtype=torch.float16, device="cuda")
        rows = _sample_rows(m.N, rows_per_mat if m.name != "lm_head" else 4 * rows_per_mat, i)
        Wr = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
        del W
        ent.append((c, s, z, x, y, m.N, m.K))
        keep.append((m, rows, Wr))
    wq().wq_linear_set(wq().make_linear_set(ent), len(ent), fmt)
    torch.cuda.synchronize()
    worst = 0.0
    for (c, s, z, x, y, N, K), (m, rows, Wr) in zip(ent, keep):
        packed, y_ref, bound = oracle_rows(Wr, x.cpu().numpy(), fmt)
        assert_bitexact(rows_np(c, s, z, fmt, N, K, rows), packed, f"{m.name} quantise")
        worst = max(worst, assert_within_tol(f16_np(y)[rows], y_ref, bound, m.name))
    return worst


def test_workload0_full():
    wl = workloads.WORKLOADS[0]
    W = synth.weights(896, 896, wl["sigma"], synth.sub_seed(wl["seed"], 0, 0))
    x = synth.activations(1, 896, synth.sub_seed(wl["seed"], 0, 1))[0]
    c, s, z = quantize_gpu(W.cuda(), "int4")
    y = torch.empty(896, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x.cuda(), c, s, z, "int4", 896, 896, y)
    packed, y_ref, bound = oracle_rows(W.numpy(), x.numpy(), "int4")
    assert_bitexact(rows_np(c, s, z, "int4", 896, 896), packed, "workload 0")
    assert_within_tol(f16_np(y), y_ref, bound, "workload 0")


def test_workload1_full_set_sampled():
    _check_set_sampled(1)


@pytest.mark.parametrize("fmt", FMTS)
def test_workload2_lm_head_sampled(fmt):
    wl = workloads.WORKLOADS[2]
    N, K = 151936, 896
    seed = synth.sub_seed(wl["seed"], 0, 0)
    W = synth.weights_with_outliers(N, K, wl["sigma"], seed, wl["outlier_frac"],
                                    wl["outlier_gain"], device="cuda")
    x = synth.activations(1, K, synth.sub_seed(wl["seed"], 0, 1), device="cuda")[0]
    c, s, z = quantize_gpu(W, fmt)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x, c, s, z, fmt, N, K, y)
    out = synth.outlier_rows(N, wl["outlier_frac"], seed).numpy()
    rows = _sample_rows(N, 3000, 7, extra=out[:200].tolist())
    Wr = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    packed, y_ref, bound = oracle_rows(Wr, x.cpu().numpy(), fmt)
    assert_bitexact(rows_np(c, s, z, fmt, N, K, rows), packed, f"lm_head {fmt}")
    assert_within_tol(f16_np(y)[rows], y_ref, bound, f"lm_head {fmt}")


def test_workload3_full_set_sampled():
    _check_set_sampled(3, rows_per_mat=16)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M", [2, 4, 8, 16, 64, 512, 2048])
def test_workload4_batch_sweep_sampled(M):
    wl = workloads.WORKLOADS[4]
    mats = [m for m in workloads.workload_mats(4) if m.name in ("l0.q", "l0.k", "l0.down", "lm_head")]
    for i, m in enumerate(mats):
        W = synth.weights(m.N, m.K, wl["sigma"], synth.sub_seed(wl["seed"], i, 0), device="cuda")
        X = synth.activations(M, m.K, synth.sub_seed(wl["seed"], i, 1), device="cuda")
        c, s, z = quantize_gpu(W, "int4")
        Y = torch.empty(M, m.N, dtype=torch.float16, device="cuda")
        wq().wq_gemm(X, M, c, s, z, "int4", m.N, m.K, Y)
        rows = _sample_rows(m.N, 24, i)
        mrows = _sample_rows(M, 16, i + 1)
        Wr = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
        _, y_ref, bound = oracle_rows(Wr, X[torch.as_tensor(mrows, device="cuda")].cpu().numpy(), "int4")
        got = f16_np(Y)[np.ix_(mrows, rows)]
        assert_within_tol(got, y_ref, bound, f"gemm M={M} {m.name}")


def test_workload4_full_set_m512_sampled():
    """The prefill-sized batch over the whole 0.5B set in one call, as the bench times it."""
    wl = workloads.WORKLOADS[4]
    M = 512
    mats = workloads.workload_mats(1)
    ent, keep = [], []
    for i, m in enumerate(mats):
        W = synth.weights(m.N, m.K, wl["sigma"], synth.sub_seed(wl["seed"], i, 0), device="cuda")
        c, s, z = quantize_gpu(W, "int4")
        X = synth.activations(M, m.K, synth.sub_seed(wl["seed"], i, 1), device="cuda")
        Y = torch.empty(M, m.N, dtype=torch.float16, device="cuda")
        rows = _sample_rows(m.N, 4, i)
        Wr = W[torch.as_tensor(rows, device="cuda")].cpu().numpy()
        del W
        ent.append((c, s, z, X, Y, m.N, m.K, M))
        keep.append((m, rows, Wr))
    wq().wq_linear_set(wq().make_linear_set(ent), len(ent), "int4")
    torch.cuda.synchronize()
    for i, ((c, s, z, X, Y, N, K, _), (m, rows, Wr)) in enumerate(zip(ent, keep)):
        mrows = _sample_rows(M, 3, 1000 + i)
        _, y_ref, bound = oracle_rows(Wr, X[torch.as_tensor(mrows, device="cuda")].cpu().numpy(), "int4")
        got = f16_np(Y)[np.ix_(mrows, rows)]
        assert_within_tol(got, y_ref, bound, f"set M=512 {m.name}")
