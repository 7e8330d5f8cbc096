"""Helpers shared by the GPU parity tests: run the CUDA path, bring results to numpy."""
import numpy as np
import torch

from oracle import wq_oracle as O

TOL = 2e-3  # |y_gpu - y_ref| <= TOL * sum_k |x_k w_hat_nk|, per output element


def wq():
    from bit_weight_quantized_unpack_b200 import wq as _wq
    return _wq


def quantize_gpu(W_dev: torch.Tensor, fmt: str):
    """wq_quantize on a device fp32 [N, K] tensor -> (codes, scale, zero) device tensors."""
    N, K = W_dev.shape
    lib = wq()
    codes, scale, zero = lib.alloc_packed(N, K, fmt)
    lib.wq_quantize(W_dev, N, K, fmt, 128, codes, scale, zero)
    return codes, scale, zero


def rows_np(codes, scale, zero, fmt, N, K, rows=None):
    """Device packed tensors -> numpy arrays in the oracle's shapes (optionally some rows)."""
    G = K // 128
    c = codes.view(N, -1)
    s = scale.view(N, G)
    z = None if zero is None else zero.view(N, G)
    if rows is not None:
        idx = torch.as_tensor(rows, device=codes.device)
        c, s = c[idx], s[idx]
        z = None if z is None else z[idx]
    c = c.cpu().numpy()
    if fmt != "ternary":
        c = c.view(np.uint32)
    s = s.cpu().numpy().view(np.uint16)
    z = None if z is None else z.cpu().numpy().view(np.uint16)
    return c, s, z


def assert_bitexact(gpu, ref, what):
    gc, gs, gz = gpu
    rc, rs, rz = ref
    assert gc.shape == rc.shape, what
    bad = np.argwhere(gc != rc)
    assert bad.size == 0, f"{what}: codes differ at {bad[:5].tolist()}"
    assert np.array_equal(gs, rs), f"{what}: scale differs at {np.argwhere(gs != rs)[:5].tolist()}"
    if rz is not None:
        assert np.array_equal(gz, rz), f"{what}: zero differs at {np.argwhere(gz != rz)[:5].tolist()}"


def assert_within_tol(y_gpu, y_ref, bound, what):
    y = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y - y_ref)
    lim = TOL * bound
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst "
                           f"err/bound {np.max(err / np.maximum(bound, 1e-300)):.3e}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0


def f16_np(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().astype(np.float64)


def oracle_rows(W_rows_np, x_np, fmt):
    """Oracle quantisation of some weight rows and the product with x ([M, K] or [K])."""
    p, s, z = O.quantize(W_rows_np, fmt)
    y, bound = O.gemv_packed(x_np, fmt, p, s, z, W_rows_np.shape[1])
    return (p, s, z), y, bound
