"""CPU ORACLE for MXFP4 block-sparse attention (UOS scaling + PNQ).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg import this module.  It shares no code with the CUDA path.

Source: [MX] "MXAttention: Data-Free Optimal Scaling and Pre-Normalization
Quantization for MXFP4 Attention", abstract (as listed on an author page).
The abstract fixes three facts:
  * the attention runs in MXFP4: elements are FP4 values that share a
    power-of-two scale per small block (the OCP microscaling format);
  * Universal Optimal Scaling (UOS) picks each block's power-of-two scale
    against the boundary Qmax = 7.25 instead of the OCP rule;
  * Pre-Normalization Quantization (PNQ) quantizes the softmax exponentials
    BEFORE normalization, and the row sum is taken over the quantized values,
    so the weights that multiply V sum to one by construction.
Everything else is a reading (R19-R22, listed with the design notes):
  R19  element format E2M1 (1 sign, 2 exponent bits with bias 1, 1 mantissa
       bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), block size 32, shared scale
       2^e with e an integer (E8M0); rounding to nearest, ties to the even code,
       magnitudes beyond 6 saturate to 6.
  R20  UOS: e = ceil(log2(amax / Qmax)), the smallest power of two that puts
       the block's largest magnitude at or below Qmax; an all-zero block has
       e = 0.  The OCP rule (e = floor(log2(amax)) - 2) is kept beside it for
       comparison only.
  R21  groups run along each product's reduction dimension: Q and K rows in
       32-element groups along D (for Q K^T); V and P in groups of 32 key rows
       counted from the first row of each key block (for P V), so no group
       crosses a block boundary; the rows past the dense prefix end in the last
       prefix block belong to no group (they are not keys of that block).
  R22  the exponentials are taken against an integer in log2 units,
       m = ceil(max_j s_j * log2(e)) over the row's keys.  Because UOS scales
       are powers of two, quantizing 2^(x - m) and 2^(x - m') gives results
       that differ exactly by 2^(m' - m) for any integers m, m', so P V / l does
       not depend on which integer is used, and a streaming kernel that only
       knows a running maximum (rounded up to an integer) computes the same
       value as one that knows the final maximum.

Pins live in tests/test_oracle_mx.py: the E2M1 table against its bit layout,
rounding ties, the UOS bound and boundary, grid values as fixed points, PNQ
normalization, the integer-shift invariance of R22, reduction to the float64
attention of rainfusion.attend_query_block when quantization is disabled, an
element-by-element loop on a tiny case, and a hand-built grouping example with
a partial prefix block.
"""
from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np

from . import rainfusion as rfo

MX_BLOCK = 32            # R19: elements per shared scale
QMAX_UOS = 7.25          # [MX] abstract: the UOS scaling boundary
E2M1_MAX = 6.0           # largest E2M1 magnitude (0.11.1)
LOG2E = 1.0 / math.log(2.0)


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code: bit 3 sign, bits 2-1 exponent (bias 1), bit 0
    mantissa; exponent field 0 is subnormal (mantissa x 0.5)."""
    sign = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return sign * 0.5 * m
    return sign * (1.0 + 0.5 * m) * 2.0 ** (e - 1)


_E2M1_POS = np.array([e2m1_value(c) for c in range(8)], dtype=np.float64)  # codes 0..7, increasing


def e2m1_round_codes(x: np.ndarray) -> np.ndarray:
    """uint8 E2M1 codes (0..15) of x: nearest representable magnitude, ties to the
    even code, saturation at 6, the sign bit from the sign of x."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E2M1_MAX)
    hi = np.clip(np.searchsorted(_E2M1_POS, a, side="left"), 0, 7)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E2M1_POS[lo]
    d_hi = _E2M1_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return code | np.where(np.signbit(x), np.uint8(0x8), np.uint8(0))


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    mag = _E2M1_POS[codes & 0x7]
    return np.where(codes & 0x8, -mag, mag)


def uos_exponent(amax: float, qmax: float = QMAX_UOS) -> int:
    """R20: the smallest integer e with amax / 2^e <= qmax (0 for amax = 0)."""
    if amax == 0.0:
        return 0
    e = math.ceil(math.log2(amax / qmax))
    # guard the log against rounding: enforce the defining inequality exactly
    while amax / 2.0 ** e > qmax:
        e += 1
    while e > -1074 and amax / 2.0 ** (e - 1) <= qmax:
        e -= 1
    return e


def ocp_exponent(amax: float) -> int:
    """The OCP MX rule, for comparison: floor(log2(amax)) minus E2M1's top exponent (2)."""
    if amax == 0.0:
        return 0
    e = math.floor(math.log2(amax))
    while 2.0 ** e > amax:
        e -= 1
    while 2.0 ** (e + 1) <= amax:
        e += 1
    return e - 2


def uos_exponents(amax: np.ndarray) -> np.ndarray:
    """uos_exponent of every element of amax (int64), with the same exact fix-ups."""
    a = np.asarray(amax, dtype=np.float64)
    e = np.zeros(a.shape, dtype=np.int64)
    nz = a > 0
    e[nz] = np.ceil(np.log2(a[nz] / QMAX_UOS)).astype(np.int64)
    up = nz & (a / np.exp2(e) > QMAX_UOS)
    e[up] += 1
    down = nz & (a / np.exp2(e - 1) <= QMAX_UOS)
    e[down] -= 1
    return e


def quantize_groups(x: np.ndarray) -> np.ndarray:
    """Every row of x is one MX group (at most 32 values): E2M1(x / 2^e) * 2^e with
    e the row's UOS exponent."""
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return x.copy()
    s = np.exp2(uos_exponents(np.max(np.abs(x), axis=-1, keepdims=True)))
    return e2m1_decode(e2m1_round_codes(x / s)) * s


def quantize_group(x: np.ndarray, rule: str = "uos") -> np.ndarray:
    """One MX group (<= 32 values) quantized and dequantized: E2M1(x / 2^e) * 2^e."""
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return x.copy()
    if rule == "uos":
        return quantize_groups(x[None])[0]
    e = ocp_exponent(float(np.max(np.abs(x))))
    return e2m1_decode(e2m1_round_codes(x / 2.0 ** e)) * 2.0 ** e


def quantize_rows(x: np.ndarray) -> np.ndarray:
    """R21 for Q and K: every row in groups of 32 along its last axis."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    for c0 in range(0, x.shape[1], MX_BLOCK):
        out[:, c0:c0 + MX_BLOCK] = quantize_groups(x[:, c0:c0 + MX_BLOCK])
    return out


def key_groups(g: rfo.SeqGeometry, b: int) -> List[range]:
    """R21: the key rows of block b split into groups of 32 from the block's first row."""
    r = rfo.block_rows(g, b)
    return [range(s, min(s + MX_BLOCK, r.stop)) for s in range(r.start, r.stop, MX_BLOCK)]


def quantize_v(v_r: np.ndarray, g: rfo.SeqGeometry) -> np.ndarray:
    """R21 for V (one head, rows of one sequence in rearranged order): each column
    quantized in groups of 32 key rows within every key block."""
    v = np.asarray(v_r, dtype=np.float64)
    out = np.zeros_like(v)
    for b in range(g.n_blocks):
        for grp in key_groups(g, b):
            out[grp.start:grp.stop] = quantize_groups(v[grp.start:grp.stop].T).T
    return out


def quantize_head(p: rfo.Problem, x_r: np.ndarray, heads: int, along: str) -> np.ndarray:
    """Quantize a rearranged BNSD/TND tensor: along="rows" for Q/K, along="keys" for V."""
    out = np.zeros(x_r.shape, dtype=np.float64)
    for s, g in p.sequences():
        for n in range(heads):
            src = p.head_rows(x_r, s, n)
            dst = p.head_rows(out, s, n)
            dst[:] = quantize_rows(src) if along == "rows" else quantize_v(src, g)
    return out


def attend_query_block_mx(qq: np.ndarray, kq: np.ndarray, vq: np.ndarray, g: rfo.SeqGeometry,
                          qb: int, key_blocks: Sequence[int], scale: float,
                          quantize_p: bool = True, m_shift: int = 0) -> np.ndarray:
    """float64 output rows of query block qb of one head with PNQ.

    qq, kq, vq are the already quantized rows of the head (rearranged order).
    Logits s = scale * q . k in float64; x = s * log2(e); m = ceil(max x) + m_shift
    (R22; m_shift exists for the invariance pin); P = 2^(x - m), quantized per
    R21 key group with UOS when quantize_p; l = sum of the quantized P; the
    output is P V / l.
    """
    qrows = rfo.block_rows(g, qb)
    q = qq[qrows.start:qrows.stop]
    groups: List[range] = []
    for b in key_blocks:
        if b < 0:
            continue
        groups.extend(key_groups(g, int(b)))
    rows = [r for grp in groups for r in grp]
    x = (scale * (q @ kq[rows].T)) * LOG2E
    m = np.ceil(x.max(axis=1, keepdims=True)) + m_shift
    pm = np.exp2(x - m)
    if quantize_p:
        c = 0
        for grp in groups:
            n = len(grp)
            pm[:, c:c + n] = quantize_groups(pm[:, c:c + n])
            c += n
    l = pm.sum(axis=1, keepdims=True)
    return (pm @ vq[rows]) / l


def attention_mx(p: rfo.Problem, qq: np.ndarray, kq: np.ndarray, vq: np.ndarray,
                 idx: np.ndarray, num: np.ndarray, scale: float, items=None) -> dict:
    """float64 output rows for (global q-block, q-head) items on quantized inputs."""
    G = p.n1 // p.n2
    table = rfo.qblock_table(p)
    if items is None:
        items = [(t, n) for t in range(len(table)) for n in range(p.n1)]
    out = {}
    for (t, n) in items:
        s, g, b = table[t]
        row = idx[t, n, :num[t, n]]
        out[(t, n)] = attend_query_block_mx(p.head_rows(qq, s, n), p.head_rows(kq, s, n // G),
                                            p.head_rows(vq, s, n // G), g, b, row, scale)
    return out
