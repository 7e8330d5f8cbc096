"""CPU oracle for group-quantised sub-byte weights and their products with fp16 activations.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or execute this
module: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg
use it. It shares no code with the CUDA path.

It follows the Whetstone README: its "Evaluation harness" section keeps a float64
reference with no fusion or shortcuts, and trusts it over any fast kernel that disagrees;
its "Quality gates" section requires kernel output to agree with a CPU reference within
a stated tolerance. Everything is numpy in
float64. Where the pages leave a step open, the plainest reading is taken and marked
READING in the function's docstring.

Pins (tests/test_oracle_pins.py): the parameter and bytes/token tables of "The one fact
that shapes everything", bits/weight of the format tables (int4 hier-g32 4.28 on the 0.5B
set and 4.26 on the 7B set included), the 243-code base-3 round trip, the +-1 XOR/popcount identity of "Measured hardware facts", closed-form quantiser
cases, an exhaustive check of the fp16 rounding routine, and exact rational products.
Parity unpinned: nothing in the quality tables of "What the weights can actually survive"
(they need trained checkpoints).
"""
from __future__ import annotations

import numpy as np

GROUP = 128  # group size along K ("int4 g128", "int2 g128", "ternary g128" in the format tables)

# --------------------------------------------------------------------------------------
# fp16 (IEEE binary16), written out from its definition: 1 sign, 5 exponent (bias 15),
# 10 fraction bits; spacing 2^(e-10) in binade [2^e, 2^(e+1)), 2^-24 below 2^-14.
# --------------------------------------------------------------------------------------
F16_MAX = 65504.0


def f16_round(d) -> np.ndarray:
    """Nearest binary16 value to each float64 (ties to even), returned as float64.

    Direct float64 -> binary16 rounding (no detour through float32, which could round
    twice). The spacing of binary16 numbers in the binade of |d| is ulp = 2^(e-11) where
    |d| = m 2^e with m in [0.5, 1), never finer than the subnormal spacing 2^-24;
    |d| / ulp is exact (power of two), so rint() (ties to even) rounds exactly once.
    Results above the largest finite value 65504 become inf.
    """
    d = np.asarray(d, dtype=np.float64)
    a = np.abs(d)
    _, e = np.frexp(a)
    ulp = np.ldexp(1.0, np.maximum(e - 11, -24))
    r = np.rint(a / ulp) * ulp
    r = np.where(r > F16_MAX, np.inf, r)
    r = np.where(np.isnan(d), np.nan, r)
    return np.copysign(r, d)


def f16_to_bits(v) -> np.ndarray:
    """binary16 bit patterns (uint16) of float64 values that are exactly representable."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.uint32) << 15
    a = np.abs(v)
    _, e = np.frexp(a)                       # a = m 2^e, m in [0.5, 1)
    normal = a >= 2.0 ** -14
    exp_field = np.where(normal, e - 1 + 15, 0)
    frac = np.where(normal, a / np.ldexp(1.0, e - 1) - 1.0, a / 2.0 ** -14) * 1024.0
    frac = np.where(np.isfinite(a), frac, 0.0)
    bits = (exp_field.astype(np.int64) << 10) + np.rint(frac).astype(np.int64)
    bits = np.where(np.isinf(a), 0x7C00, bits)
    assert np.all(f16_round(v)[np.isfinite(v)] == v[np.isfinite(v)]), "not a binary16 value"
    return (bits.astype(np.uint32) | sign).astype(np.uint16)


def f16_from_bits(b) -> np.ndarray:
    """float64 value of binary16 bit patterns (finite and inf; NaN patterns -> nan)."""
    b = np.asarray(b, dtype=np.uint16).astype(np.int64)
    s = np.where(b & 0x8000, -1.0, 1.0)
    ex = (b >> 10) & 0x1F
    fr = (b & 0x3FF).astype(np.float64)
    val = np.where(ex == 0, fr * 2.0 ** -24, np.ldexp(1.0 + fr / 1024.0, ex - 15))
    val = np.where(ex == 31, np.where(fr == 0, np.inf, np.nan), val)
    return s * val


# --------------------------------------------------------------------------------------
# Quantisers.  Whetstone README, "What the weights can actually survive": round-to-nearest
# at group 128, with one fp16 scale and one fp16 zero per group (0.25 bits/weight of
# metadata); format table rows int4 g128 (4.25), int3 g128 (3.25), int2 g128 (2.25),
# ternary g128 (1.71).
# --------------------------------------------------------------------------------------

INT_BITS = {"int4": 4, "int3": 3, "int2": 2}

def quantize_int(W, bits: int):
    """Asymmetric round-to-nearest group-128 quantisation along K to `bits`-bit codes.

    READING (the pages name round-to-nearest, asymmetric, group 128 and fp16 scale and
    zero, but give no formula); per (row n, group g), with Q = 2^bits - 1 and w in float64:
        lo = min w, hi = max w
        s  = fp16(( hi - lo) / Q);  s = 1 if that is 0 (constant group / underflow)
        z  = clamp(rint(-lo / s), 0, Q)          (integer zero point, stored as fp16)
        q  = clamp(rint(w / s) + z, 0, Q)        (rint: ties to even)
    so that w ~ w_hat = (q - z) * s with the stored fp16 s and z.
    Returns codes uint32 [N, K*bits/32] (code k at bits bits*k .. bits*k + bits - 1 of the
    row's little-endian bit stream, word j holding stream bits 32 j .. 32 j + 31: for 2 and 4
    bits word k // (32/bits), bits bits*(k % (32/bits)); 3-bit codes may straddle two
    words), scale and zero as uint16 fp16 bits [N, K/128].
    READING for int3 (the format table gives only "int3 g128", 3.25 bits/weight): the same
    quantiser with Q = 7 and the same bit-stream order as int2 / int4.
    """
    W = np.asarray(W)
    N, K = W.shape
    assert K % GROUP == 0 and bits in (2, 3, 4)
    G = K // GROUP
    Q = float(2 ** bits - 1)
    w = W.astype(np.float64).reshape(N, G, GROUP)
    lo = w.min(axis=2)
    hi = w.max(axis=2)
    s = f16_round((hi - lo) / Q)
    s = np.where(s == 0.0, 1.0, s)
    z = np.clip(np.rint(-lo / s), 0.0, Q) + 0.0          # an integer: no negative zero
    q = np.clip(np.rint(w / s[:, :, None]) + z[:, :, None], 0.0, Q).astype(np.uint32)
    return pack_int(q.reshape(N, K), bits), f16_to_bits(s), f16_to_bits(z)


def pack_int(q, bits: int) -> np.ndarray:
    """Pack codes [N, K] (< 2^bits) into uint32 words, code k at bits bits*k.. of the row's
    little-endian bit stream (for 2 and 4 bits: word k // per, bit bits*(k % per))."""
    q = np.asarray(q, dtype=np.uint32)
    N, K = q.shape
    if 32 % bits:
        return _pack_stream(q, bits)
    per = 32 // bits
    q = q.reshape(N, K // per, per)
    words = np.zeros((N, K // per), dtype=np.uint32)
    for j in range(per):
        words |= q[:, :, j] << np.uint32(bits * j)
    return words


def _pack_stream(q, bits: int) -> np.ndarray:
    """Bit-stream packing for code widths that do not divide 32: code k's bit b goes to
    stream bit bits*k + b, i.e. word (bits*k + b) // 32, bit (bits*k + b) % 32."""
    N, K = q.shape
    assert (K * bits) % 32 == 0
    words = np.zeros((N, K * bits // 32), dtype=np.uint64)
    for k in range(K):
        pos = bits * k
        j, off = divmod(pos, 32)
        v = q[:, k].astype(np.uint64) << np.uint64(off)        # up to 34 bits
        words[:, j] |= v & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[:, j + 1] |= v >> np.uint64(32)
    return words.astype(np.uint32)


def _unpack_stream(codes, bits: int, K: int) -> np.ndarray:
    """Inverse of _pack_stream."""
    codes = np.asarray(codes, dtype=np.uint32).astype(np.uint64)
    N = codes.shape[0]
    out = np.empty((N, K), dtype=np.int64)
    mask = np.uint64(2 ** bits - 1)
    for k in range(K):
        j, off = divmod(bits * k, 32)
        v = codes[:, j] >> np.uint64(off)
        if off + bits > 32:
            v |= codes[:, j + 1] << np.uint64(32 - off)
        out[:, k] = (v & mask).astype(np.int64)
    return out


def unpack_int(codes, bits: int, K: int) -> np.ndarray:
    """Inverse of pack_int: uint32 words [N, K*bits/32] -> codes int64 [N, K]."""
    if 32 % bits:
        return _unpack_stream(codes, bits, K)
    codes = np.asarray(codes, dtype=np.uint32)
    N = codes.shape[0]
    per = 32 // bits
    mask = np.uint32(2 ** bits - 1)
    out = np.empty((N, K // per, per), dtype=np.int64)
    for j in range(per):
        out[:, :, j] = (codes >> np.uint32(bits * j)) & mask
    return out.reshape(N, K)


def dequant_int(codes, scale_bits, zero_bits, bits: int, K: int) -> np.ndarray:
    """w_hat[n, k] = (q - z) * s, float64, with the stored fp16 s and z of k's group."""
    q = unpack_int(codes, bits, K).astype(np.float64)
    s = np.repeat(f16_from_bits(scale_bits), GROUP, axis=1)
    z = np.repeat(f16_from_bits(zero_bits), GROUP, axis=1)
    return (q - z) * s


# Ternary.  TKintegers K5, "What is K5?": a one-byte code made of five balanced-ternary
# digits, so 243 values (trits, not bits).  READING: the byte holds five
# ternary WEIGHTS t_0..t_4 in {-1, 0, +1} as the base-3 number sum_i (t_i + 1) 3^i, lowest
# weight in the least significant digit.
TRITS_PER_BYTE = 5
TERNARY_GROUP_BYTES = -(-GROUP // TRITS_PER_BYTE)  # 26: 25 full bytes + one with 3 trits


def trits_to_byte(t5) -> int:
    """Five trits (t_0 first) -> one byte sum_i (t_i + 1) 3^i in 0..242."""
    assert len(t5) == TRITS_PER_BYTE and all(t in (-1, 0, 1) for t in t5)
    return sum((int(t) + 1) * 3 ** i for i, t in enumerate(t5))


def byte_to_trits(b: int) -> tuple[int, ...]:
    """One byte 0..242 -> its five trits (t_0 first); bytes 243..255 are not codes."""
    if not 0 <= b <= 242:
        raise ValueError(f"byte {b} is not a base-3 code (valid: 0..242)")
    out = []
    for _ in range(TRITS_PER_BYTE):
        out.append(b % 3 - 1)
        b //= 3
    return tuple(out)


def quantize_ternary(W):
    """Ternary {-1, 0, +1} group-128 quantisation with an fp16 absmean scale.

    READING (format table row "ternary g128", absmean scale): per (row, group)
        a = (sum_k |w_k|) / 128   -- float64, summed in increasing k order
        s = fp16(a);  s = 1 if that is 0
        t = clamp(rint(w / s), -1, 1)
    Packing: each group's 128 trits fill 26 bytes, five per byte as trits_to_byte; the
    last byte holds trits 125..127 and two pad trits of value 0 (digit 1). Groups follow
    each other along the row. Returns packed uint8 [N, 26*K/128], scale uint16 [N, K/128].
    """
    W = np.asarray(W)
    N, K = W.shape
    assert K % GROUP == 0
    G = K // GROUP
    w = W.astype(np.float64).reshape(N, G, GROUP)
    acc = np.zeros((N, G), dtype=np.float64)
    for k in range(GROUP):                     # the sum's order is part of the definition
        acc += np.abs(w[:, :, k])
    s = f16_round(acc / GROUP)
    s = np.where(s == 0.0, 1.0, s)
    t = np.clip(np.rint(w / s[:, :, None]), -1.0, 1.0).astype(np.int64)
    return pack_ternary(t.reshape(N, K)), f16_to_bits(s)


def pack_ternary(t) -> np.ndarray:
    """Trits [N, K] -> bytes [N, 26*K/128] (see quantize_ternary for the layout)."""
    t = np.asarray(t, dtype=np.int64)
    N, K = t.shape
    G = K // GROUP
    pad = TERNARY_GROUP_BYTES * TRITS_PER_BYTE - GROUP          # 2 pad trits per group
    tg = np.concatenate([t.reshape(N, G, GROUP), np.zeros((N, G, pad), np.int64)], axis=2)
    d = (tg + 1).reshape(N, G, TERNARY_GROUP_BYTES, TRITS_PER_BYTE)
    byte = np.zeros((N, G, TERNARY_GROUP_BYTES), dtype=np.int64)
    for i in range(TRITS_PER_BYTE):
        byte += d[..., i] * 3 ** i
    return byte.reshape(N, G * TERNARY_GROUP_BYTES).astype(np.uint8)


def unpack_ternary(packed, K: int) -> np.ndarray:
    """Inverse of pack_ternary: bytes [N, 26*K/128] -> trits int64 [N, K]."""
    p = np.asarray(packed, dtype=np.int64)
    N = p.shape[0]
    G = K // GROUP
    if np.any(p > 242):
        raise ValueError("packed ternary data holds a byte above 242")
    p = p.reshape(N, G, TERNARY_GROUP_BYTES)
    d = np.empty((N, G, TERNARY_GROUP_BYTES, TRITS_PER_BYTE), dtype=np.int64)
    for i in range(TRITS_PER_BYTE):
        d[..., i] = p % 3
        p = p // 3
    t = d.reshape(N, G, TERNARY_GROUP_BYTES * TRITS_PER_BYTE)[:, :, :GROUP] - 1
    return t.reshape(N, K)


def dequant_ternary(packed, scale_bits, K: int) -> np.ndarray:
    """w_hat[n, k] = t * s, float64."""
    t = unpack_ternary(packed, K).astype(np.float64)
    return t * np.repeat(f16_from_bits(scale_bits), GROUP, axis=1)


# --------------------------------------------------------------------------------------
# Hierarchical int4, group 32.  Whetstone README, "What the weights can actually survive":
# group 32 with an fp16 scale and zero per group would cost 1.0 bits/weight of metadata,
# so the format stores two 4-bit indices per group against one f16 pair per row (format
# table of "The one fact that shapes everything": "int4 hier-g32", 4.28 bits/weight);
# "Prior art": the same idea as GGUF Q4_K, sub-block scale and min indices against a
# super-block f16 pair; "New in 0.6.0": the shared fp16 row scale could underflow to zero
# and garble whole rows (seen only on the 7B model).
# --------------------------------------------------------------------------------------
HIER_GROUP = 32
F16_TINY = 2.0 ** -24  # smallest positive binary16


def _row_scale(num):
    """fp16(num / 15) for the row pair, with the underflow guard: a positive numerator whose
    quotient rounds to 0 gives the smallest positive binary16 instead, and a zero numerator
    (nothing to scale) gives 1."""
    d = f16_round(num / 15.0)
    d = np.where((d == 0.0) & (num > 0.0), F16_TINY, d)
    return np.where(num == 0.0, 1.0, d)


def quantize_int4h(W):
    """Hierarchical int4 quantisation: 4-bit codes in groups of 32 along K, each group's
    scale and min given by two 4-bit indices into one fp16 pair (d, dm) per row.

    READING (the pages give the geometry -- group 32, two 4-bit indices per group, an f16
    pair per row -- and the Q4_K analogy, not a formula). Round to nearest throughout, per
    row n, in float64:
        per group g (32 consecutive k):  lo = min w, hi = max w
            m_g = max(0, -lo)                the group's min offset (Q4_K style, never < 0)
            s_g = (hi + m_g) / 15            the step that spans [-m_g, hi]
        d  = fp16(max_g s_g / 15),  dm = fp16(max_g m_g / 15)      (with _row_scale's guard)
        a_g = clamp(rint(s_g / d), 0, 15),   b_g = clamp(rint(m_g / dm), 0, 15)
        S_g = d a_g,  Z_g = dm b_g           (exact: an fp16 value times a 4-bit integer)
        q   = clamp(rint((w + Z_g) / S_g), 0, 15)   (q = 0 where S_g = 0)
    and w_hat = S_g q - Z_g. rint is ties-to-even; w + Z_g and the quotients are float64
    operations, rounded once each, in this order.
    Returns codes uint32 [N, K/8] (the int4 layout: code k in word k/8, bits 4(k%8)),
    pair uint16 [N, 2] (fp16 bits of d, dm) and idx uint8 [N, K/32] (a_g | b_g << 4).
    """
    W = np.asarray(W)
    N, K = W.shape
    assert K % GROUP == 0
    G = K // HIER_GROUP
    w = W.astype(np.float64).reshape(N, G, HIER_GROUP)
    lo = w.min(axis=2)
    hi = w.max(axis=2)
    m = np.maximum(0.0, -lo)
    s = (hi + m) / 15.0
    d = _row_scale(s.max(axis=1))
    dm = _row_scale(m.max(axis=1))
    a = np.clip(np.rint(s / d[:, None]), 0.0, 15.0)
    b = np.clip(np.rint(m / dm[:, None]), 0.0, 15.0)
    S = d[:, None] * a
    Z = dm[:, None] * b
    safe = np.where(S > 0.0, S, 1.0)
    q = np.clip(np.rint((w + Z[:, :, None]) / safe[:, :, None]), 0.0, 15.0)
    q = np.where((S > 0.0)[:, :, None], q, 0.0).astype(np.uint32)
    pair = np.stack([f16_to_bits(d), f16_to_bits(dm)], axis=1)
    idx = (a.astype(np.uint32) | (b.astype(np.uint32) << 4)).astype(np.uint8)
    return pack_int(q.reshape(N, K), 4), pair, idx


def dequant_int4h(codes, pair_bits, idx, K: int) -> np.ndarray:
    """w_hat[n, k] = d_n a_g q - dm_n b_g for k in group g (float64, exact)."""
    q = unpack_int(codes, 4, K).astype(np.float64)
    pr = f16_from_bits(np.asarray(pair_bits, dtype=np.uint16))
    ix = np.asarray(idx, dtype=np.int64)
    S = pr[:, 0:1] * (ix & 15).astype(np.float64)
    Z = pr[:, 1:2] * (ix >> 4).astype(np.float64)
    return q * np.repeat(S, HIER_GROUP, axis=1) - np.repeat(Z, HIER_GROUP, axis=1)


def int4h_bytes(N: int, K: int) -> int:
    """Stored bytes of an [N, K] int4h weight: codes + one index byte per 32 + fp16 pair per row."""
    return N * K // 2 + N * K // HIER_GROUP + 4 * N


# --------------------------------------------------------------------------------------
# The product.  Whetstone README, "The one fact that shapes everything": at batch 1 every
# weight is read once and used for one multiply-add; "Evaluation harness": float64
# throughout.  y = x . w_hat^T, with the fp16 activations taken as exact float64 values.
# --------------------------------------------------------------------------------------

def linear(x, w_hat):
    """y[m, n] = sum_k x[m, k] w_hat[n, k] and bound[m, n] = sum_k |x[m, k] w_hat[n, k]|.

    x: fp16 (or float64) [M, K] or [K]; w_hat float64 [N, K]. A float64 matrix product
    (library primitive) is the sum. The bound is the scale of the acceptance test
    |y_gpu - y| <= 2e-3 * bound.
    """
    xd = np.asarray(x).astype(np.float64)
    y = xd @ w_hat.T
    bound = np.abs(xd) @ np.abs(w_hat).T
    return y, bound


def gemv_packed(x, fmt: str, packed, scale_bits, zero_bits, K: int):
    """Dequantise packed weights, then linear(); fmt in {'int4', 'int3', 'int2', 'ternary',
    'int4h'} (for 'int4h' scale_bits is the row pair and zero_bits the index bytes)."""
    if fmt == "ternary":
        w_hat = dequant_ternary(packed, scale_bits, K)
    elif fmt == "int4h":
        w_hat = dequant_int4h(packed, scale_bits, zero_bits, K)
    else:
        w_hat = dequant_int(packed, scale_bits, zero_bits, INT_BITS[fmt], K)
    return linear(x, w_hat)


def quantize(W, fmt: str):
    """Dispatch: returns (packed, scale_bits, zero_bits or None)."""
    if fmt == "ternary":
        p, s = quantize_ternary(W)
        return p, s, None
    if fmt == "int4h":
        return quantize_int4h(W)
    return quantize_int(W, INT_BITS[fmt])


# --------------------------------------------------------------------------------------
# Head rescoring.  Whetstone README, feature list (--head-rescore): an fp16 copy of the
# output projection is kept, and only the logits that decide the token are recomputed
# from it.  READING: the logits that decide the token are the k largest quantised-head
# logits (ties to the lower row); each is recomputed as the product of x with the fp16
# row, and the token is the row with the largest recomputed logit (ties to the lower row).
# --------------------------------------------------------------------------------------

def topk_rows(y, k: int) -> np.ndarray:
    """Rows of the k largest values of y (1-D), largest first, equal values by lower row.

    A stable sort on the negated values is the definition written out: numpy's stable
    argsort keeps equal keys in index order. k is clipped to len(y)."""
    yd = np.asarray(y, dtype=np.float64)
    order = np.argsort(-yd, kind="stable")
    return order[: min(k, len(yd))].astype(np.int64)


def rescore(x, w16_rows) -> tuple[np.ndarray, np.ndarray]:
    """The candidates' logits from the fp16 head: linear() of x with the given fp16 rows.

    Returns (logits, bound), float64, for the acceptance test |l_gpu - l| <= 2e-3 bound."""
    w = np.asarray(w16_rows).astype(np.float64)
    return linear(np.asarray(x).reshape(-1), w)


def pick_token(rows, logits) -> int:
    """The row with the largest logit among the candidates; equal logits: the lower row."""
    rows = np.asarray(rows, dtype=np.int64)
    lg = np.asarray(logits, dtype=np.float64)
    best = lg.max()
    return int(rows[lg == best].min())


# --------------------------------------------------------------------------------------
# Whetstone README, "Measured hardware facts": for a, b in {-1,+1}^K packed as bits
# {1, 0}, dot(a, b) = K - 2 popcount(a XOR b).
# --------------------------------------------------------------------------------------

def pm1_dot_popcount(a_bits: int, b_bits: int, K: int) -> int:
    """dot of two +-1 vectors given as K-bit integers (bit i = 1 means +1)."""
    return K - 2 * bin((a_bits ^ b_bits) & ((1 << K) - 1)).count("1")


def ternary_pm1_dot_popcount(a_bits: int, trits) -> int:
    """sum_i a_i t_i for +-1 a (bits as above) and trits t, by the identity on t's support.

    On the support S = {i : t_i != 0}, t is itself a +-1 vector, so the identity applies
    to the bits restricted to S: dot = |S| - 2 popcount((a XOR t_plus) AND S).
    """
    support = sum(1 << i for i, t in enumerate(trits) if t != 0)
    t_plus = sum(1 << i for i, t in enumerate(trits) if t == 1)
    return bin(support).count("1") - 2 * bin((a_bits ^ t_plus) & support).count("1")


# --------------------------------------------------------------------------------------
# Roofline and byte accounting.  Whetstone README, "The one fact that shapes everything":
# tok/s_ceiling = bandwidth / bytes_read_per_token, over the blocks and the tied lm_head.
# --------------------------------------------------------------------------------------

def set_params(mats) -> tuple[int, int, int]:
    """(transformer-block weights, lm_head weights, total) of a layer set."""
    head = sum(m.N * m.K for m in mats if m.name == "lm_head")
    total = sum(m.N * m.K for m in mats)
    return total - head, head, total


def bytes_per_token(params: int, bits_per_weight: float) -> float:
    return params * bits_per_weight / 8.0


def tok_s_ceiling(bandwidth_bytes_per_s: float, bytes_per_token_: float) -> float:
    return bandwidth_bytes_per_s / bytes_per_token_


def stored_bits_per_weight(fmt: str, K: int | None = None) -> float:
    """Bits per weight of this layout as stored: codes + fp16 metadata per 128 weights
    (int4h: codes + one index byte per 32 weights + one fp16 pair per row of K)."""
    if fmt == "int4h":
        return 4 + 8 / HIER_GROUP + 32 / K
    if fmt == "ternary":
        return (TERNARY_GROUP_BYTES * 8 + 16) / GROUP
    return INT_BITS[fmt] + 32 / GROUP
