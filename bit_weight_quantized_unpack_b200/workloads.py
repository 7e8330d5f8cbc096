"""Shapes of the synthetic workloads (no arithmetic of the method lives here).

The layer sets are the linear layers that one decoded token reads, as the Whetstone
README counts them in "The one fact that shapes everything" (parameter table: transformer
blocks plus the tied lm_head of Qwen2.5-0.5B). Each entry is (name, N, K): the weight is
[N, K] (out_features x in_features) and y = x . W^T.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Linear:
    name: str
    N: int  # output rows
    K: int  # reduction length (in_features)


def decoder_set(layers: int, hidden: int, kv: int, inter: int, vocab: int) -> list[Linear]:
    """Per layer q, k, v, o, gate, up, down, then the output projection (lm_head)."""
    out: list[Linear] = []
    for i in range(layers):
        out += [
            Linear(f"l{i}.q", hidden, hidden),
            Linear(f"l{i}.k", kv, hidden),
            Linear(f"l{i}.v", kv, hidden),
            Linear(f"l{i}.o", hidden, hidden),
            Linear(f"l{i}.gate", inter, hidden),
            Linear(f"l{i}.up", inter, hidden),
            Linear(f"l{i}.down", hidden, inter),
        ]
    out.append(Linear("lm_head", vocab, hidden))
    return out


def qwen05b_set() -> list[Linear]:
    """Qwen2.5-0.5B: 24 layers, hidden 896, 2 kv heads x 64, MLP 4864, vocab 151936."""
    return decoder_set(24, 896, 128, 4864, 151936)


def qwen7b_set() -> list[Linear]:
    """Qwen2.5-7B: 28 layers, hidden 3584, 4 kv heads x 128, MLP 18944, vocab 152064."""
    return decoder_set(28, 3584, 512, 18944, 152064)


# The five workloads. Sigma is the standard deviation of the synthetic fp32 weights;
# x is N(0, 1) rounded to fp16. Seeds are 1000 + workload index.
WORKLOADS = {
    0: dict(name="single_896x896_int4", sigma=0.02, seed=1000,
            mats=[Linear("w", 896, 896)], fmts=("int4",), M=(1,)),
    1: dict(name="qwen2.5-0.5b_decode_set_int4", sigma=0.02, seed=1001,
            mats=None, fmts=("int4",), M=(1,)),
    2: dict(name="lm_head_151936x896_sweep", sigma=0.02, seed=1002,
            mats=[Linear("lm_head", 151936, 896)], fmts=("int4", "int2", "ternary"), M=(1,),
            outlier_frac=0.01, outlier_gain=8.0),
    3: dict(name="qwen2.5-7b_decode_set_int4", sigma=0.015, seed=1003,
            mats=None, fmts=("int4",), M=(1,)),
    4: dict(name="qwen2.5-0.5b_set_batch_sweep_int4", sigma=0.02, seed=1004,
            mats=None, fmts=("int4",), M=(1, 2, 4, 8, 16, 64, 512, 2048)),
}


def workload_mats(idx: int) -> list[Linear]:
    w = WORKLOADS[idx]
    if w["mats"] is not None:
        return list(w["mats"])
    return qwen7b_set() if idx == 3 else qwen05b_set()
