"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module only draws random numbers: it holds none of the quantisation or product
arithmetic. Weights are fp32 N(0, sigma^2); activations are N(0, 1) rounded to fp16.
Generation uses torch's seeded generators (CPU: Mersenne Twister, CUDA: Philox), so the
same (seed, device) always gives the same tensor. Small cases are drawn on the CPU and
copied to the GPU, so both sides see identical bytes; full-size cases are drawn on the
GPU and the rows an oracle check needs are copied back.
"""
from __future__ import annotations

import torch


def sub_seed(base: int, index: int, what: int) -> int:
    """Distinct seed per (workload seed, matrix index, stream) -- what: 0 = W, 1 = x."""
    return (base * 1_000_003 + index * 7 + what) % (2**62)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weights(N: int, K: int, sigma: float, seed: int, device="cpu") -> torch.Tensor:
    """fp32 [N, K] with entries N(0, sigma^2)."""
    w = torch.randn(N, K, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return w.mul_(sigma)


def outlier_rows(N: int, frac: float, seed: int) -> torch.Tensor:
    """floor(frac * N) distinct row indices (int64, CPU), drawn by a seeded permutation."""
    n = int(frac * N)
    return torch.randperm(N, generator=_gen(seed ^ 0x5EED, "cpu"))[:n].sort().values


def weights_with_outliers(N: int, K: int, sigma: float, seed: int, frac: float, gain: float,
                          device="cpu") -> torch.Tensor:
    """As weights(), with floor(frac * N) seeded rows multiplied by gain."""
    w = weights(N, K, sigma, seed, device)
    idx = outlier_rows(N, frac, seed).to(w.device)
    w[idx] *= gain
    return w


def activations(M: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """fp16 [M, K]: N(0, 1) drawn in fp32 then rounded to fp16 by torch."""
    x = torch.randn(M, K, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch.float16)
