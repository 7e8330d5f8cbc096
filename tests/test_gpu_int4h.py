"""Hierarchical int4 (group-32 indices against a per-row fp16 pair) on the GPU.

Whetstone README, "What the weights can actually survive": groups of 32 whose scale and min
are two 4-bit indices into one f16 pair per row ("int4 hier-g32", 4.28 bits/weight), with
"New in 0.6.0"'s guard against a row scale that underflows to zero.
- The quantiser is bit-exact against the oracle (codes, pairs and index bytes), including
  rows of zeros, constant rows, rows that trigger the underflow guard, one-signed rows and
  outlier rows.
- The streaming product (M = 1 .. 4, single matrices and sets, fused argmax) is within the
  product bound of the oracle, element by element, on shapes that span several ring slots
  and end in ragged tails (N not a multiple of the 4-cell metadata unit).
- Requests outside the served range return their documented status before any launch.
"""
import numpy as np
import pytest
import torch

from bit_weight_quantized_unpack_b200 import synth, workloads

from gpu_util import assert_within_tol, f16_np, wq
from oracle import wq_oracle as O

pytestmark = pytest.mark.gpu


def quantize_h(W_dev):
    N, K = W_dev.shape
    lib = wq()
    c, s, z = lib.alloc_packed(N, K, "int4h")
    lib.wq_quantize(W_dev, N, K, "int4h", 32, c, s, z)
    return c, s, z


def to_np(c, s, z, N, K):
    return (c.view(N, -1).cpu().numpy().view(np.uint32), s.view(N, 2).cpu().numpy().view(np.uint16),
            z.view(N, K // 32).cpu().numpy())


def special_rows(K, rng_seed):
    """Rows that exercise each branch of the definition."""
    g = torch.Generator().manual_seed(rng_seed)
    rows = [
        torch.zeros(K),                              # nothing to scale: d = dm = 1, all codes 0
        torch.full((K,), 0.0123),                    # constant positive: m_g = 0 everywhere
        torch.full((K,), -0.5),                      # constant negative: s_g = 0 after the min
        torch.randn(K, generator=g) * 1e-9,          # tiny: fp16(max s / 15) underflows -> 2^-24
        torch.rand(K, generator=g) * 0.1,            # one-signed (positive)
        -torch.rand(K, generator=g) * 0.1,           # one-signed (negative)
        torch.randn(K, generator=g) * 0.02,
    ]
    r = torch.randn(K, generator=g) * 0.02           # one outlier group
    r[32:64] *= 40.0
    rows.append(r)
    return torch.stack(rows).float()


@pytest.mark.parametrize("N,K", [(263, 896), (64, 4864), (5, 128), (33, 2048)])
def test_quantizer_bitexact(N, K):
    W = synth.weights(N, K, 0.02, seed=700 + N)
    W[: min(N, 8)] = special_rows(K, 701)[: min(N, 8)]
    c, s, z = quantize_h(W.cuda())
    torch.cuda.synchronize()
    gc, gs, gz = to_np(c, s, z, N, K)
    rc, rs, rz = O.quantize(W.numpy(), "int4h")
    assert np.array_equal(gs, rs), f"pairs differ at rows {np.argwhere((gs != rs).any(1))[:5].ravel()}"
    assert np.array_equal(gz, rz), f"index bytes differ at {np.argwhere(gz != rz)[:5].tolist()}"
    assert np.array_equal(gc, rc), f"codes differ at {np.argwhere(gc != rc)[:5].tolist()}"
    if N >= 4:
        assert gs[3, 0] == 0x0001, "underflow guard: tiny row's d must be the smallest binary16"


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(263, 896), (1029, 4864), (6, 128), (130, 18944)])
def test_gemm_small_m(M, N, K):
    W = synth.weights(N, K, 0.02, seed=710 + N + K)
    W[: min(N, 8)] = special_rows(K, 711)[: min(N, 8)]
    X = synth.activations(M, K, seed=712 + M)
    c, s, z = quantize_h(W.cuda())
    Y = torch.empty(M, N, dtype=torch.float16, device="cuda")
    if M == 1:
        wq().wq_gemv(X[0].cuda(), c, s, z, "int4h", N, K, Y[0])
    else:
        wq().wq_gemm(X.cuda(), M, c, s, z, "int4h", N, K, Y)
    torch.cuda.synchronize()
    p, pr, ix = to_np(c, s, z, N, K)
    y_ref, bound = O.gemv_packed(X.numpy(), "int4h", p, pr, ix, K)
    assert_within_tol(f16_np(Y), y_ref, bound, f"int4h M={M} {N}x{K}")
    assert wq().wq_device_errors(clear=True) == 0


def test_decode_set_and_argmax():
    """The 0.5B decode set's distinct layer shapes, as one int4h set, then the lm_head-shaped
    product with the fused argmax (ties to the lowest row)."""
    mats = workloads.workload_mats(1)
    shapes = []
    for m in mats:
        if (m.N, m.K) not in shapes:
            shapes.append((m.N, m.K))
    lib = wq()
    ent, refs = [], []
    for i, (N, K) in enumerate(shapes):
        if N > 20000:
            N = 4099  # lm_head-shaped K with fewer rows: the oracle stays fast
        W = synth.weights(N, K, 0.02, seed=720 + i)
        x = synth.activations(1, K, seed=730 + i)[0]
        c, s, z = quantize_h(W.cuda())
        y = torch.empty(N, dtype=torch.float16, device="cuda")
        ent.append((c, s, z, x.cuda(), y, N, K))
        refs.append((W, x))
    lib.wq_linear_set(lib.make_linear_set(ent), len(ent), "int4h")
    torch.cuda.synchronize()
    for (c, s, z, _, y, N, K), (W, x) in zip(ent, refs):
        p, pr, ix = to_np(c, s, z, N, K)
        y_ref, bound = O.gemv_packed(x.numpy(), "int4h", p, pr, ix, K)
        assert_within_tol(f16_np(y), y_ref, bound, f"int4h set {N}x{K}")
        # the set's outputs equal the single product's, bit for bit
        y1 = torch.empty_like(y)
        lib.wq_gemv(x.cuda(), c, s, z, "int4h", N, K, y1)
        torch.cuda.synchronize()
        assert torch.equal(y1, y), f"set vs single {N}x{K}"
    # fused argmax on the last (lm_head-shaped) entry
    c, s, z, xd, y, N, K = ent[-1]
    ws = torch.zeros(lib.wq_argmax_workspace_bytes(), dtype=torch.uint8, device="cuda")
    am = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    y2 = torch.empty_like(y)
    lib.wq_gemv_argmax(xd, c, s, z, "int4h", N, K, y2, am, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(y2, y)
    r = int(np.argmax(y.float().cpu().numpy()))
    assert int(am.item()) == r, "argmax is the first row of the largest fp16 value"
    # a planted tie: the winning row copied into a lower row (and a higher one) -> the lowest wins
    lo_row = 0 if r > 0 else None
    for dst in ([lo_row] if lo_row is not None else []) + [N - 1]:
        if dst == r:
            continue
        c.view(N, -1)[dst] = c.view(N, -1)[r]
        s.view(N, 2)[dst] = s.view(N, 2)[r]
        z.view(N, -1)[dst] = z.view(N, -1)[r]
    lib.wq_gemv_argmax(xd, c, s, z, "int4h", N, K, y2, am, ws, ws.numel())
    torch.cuda.synchronize()
    assert int(am.item()) == (0 if lo_row is not None else r)


def test_full_size_lm_head_sampled():
    """Qwen2.5-0.5B lm_head shape (151936 x 896) at M = 1 in the launch configuration of the
    set: sampled rows against the oracle."""
    N, K = 151936, 896
    W = synth.weights(N, K, 0.02, seed=740, device="cuda")
    x = synth.activations(1, K, seed=741, device="cuda")[0]
    c, s, z = quantize_h(W)
    y = torch.empty(N, dtype=torch.float16, device="cuda")
    wq().wq_gemv(x, c, s, z, "int4h", N, K, y)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(N - 67, N),
                                     np.random.default_rng(742).integers(0, N, 512)]))
    idx = torch.as_tensor(rows, device="cuda")
    Wr = W[idx].cpu().numpy()
    rc, rs, rz = O.quantize(Wr, "int4h")
    gc, gs, gz = to_np(c.view(N, -1)[idx].reshape(-1), s.view(N, 2)[idx].reshape(-1),
                       z.view(N, -1)[idx].reshape(-1), len(rows), K)
    assert np.array_equal(gc, rc) and np.array_equal(gs, rs) and np.array_equal(gz, rz)
    y_ref, bound = O.gemv_packed(x.cpu().numpy(), "int4h", rc, rs, rz, K)
    assert_within_tol(f16_np(y[idx]), y_ref, bound, "int4h lm_head sampled rows")


def test_unsupported_and_checks():
    lib = wq()
    N, K = 64, 896
    c, s, z = quantize_h(synth.weights(N, K, 0.02, seed=750).cuda())
    X = torch.zeros(5, 32768, dtype=torch.float16, device="cuda")
    Y = torch.empty(5, N, dtype=torch.float16, device="cuda")
    with pytest.raises(lib.WQError) as e:  # M = 5
        lib.wq_gemm(X[:, :K].contiguous(), 5, c, s, z, "int4h", N, K, Y)
    assert e.value.status == lib.WQ_ERR_UNSUPPORTED
    c2, s2, z2 = lib.alloc_packed(N, 32768, "int4h")
    with pytest.raises(lib.WQError) as e:  # M * K = 4 * 32768 > 92160
        lib.wq_gemm(X[:4].contiguous(), 4, c2, s2, z2, "int4h", N, 32768, Y[:4])
    assert e.value.status == lib.WQ_ERR_UNSUPPORTED
    with pytest.raises(lib.WQError) as e:  # group must be 32
        lib.wq_quantize(torch.zeros(N, K, device="cuda"), N, K, "int4h", 128, c, s, z)
    assert e.value.status == lib.WQ_ERR_ARG
    buf = torch.empty(2 * N + 8, dtype=torch.int16, device="cuda")
    with pytest.raises(lib.WQError) as e:  # pair array at a 2-byte offset
        lib.wq_gemv(X[0, :K], c, buf[1:1 + 2 * N], z, "int4h", N, K, Y[0])
    assert e.value.status == lib.WQ_ERR_ALIGN
    torch.cuda.synchronize()
    assert lib.wq_scale_bytes("int4h", N, K) == 4 * N
    assert lib.wq_zero_bytes("int4h", N, K) == N * K // 32
    assert lib.wq_codes_bytes("int4h", N, K) == N * K // 2
