"""Pins for the oracle's FP8 E4M3 quantization (the "mix" precision reading, CPU only).

The E4M3 format is fixed by its definition (1 sign, 4 exponent bits with bias 7,
3 mantissa bits, no infinities, S.1111.111 = NaN): closed-form values, the
round-to-nearest-even rule checked at every midpoint, saturation, and an
independent conversion (PyTorch's float8_e4m3fn cast, which the oracle does not
use) on random values.
"""
import math

import numpy as np
import pytest
import torch

from oracle import rainfusion as rf


def test_e4m3_closed_forms():
    assert rf.e4m3_value(0x7E) == 448.0                 # largest finite
    assert rf.e4m3_value(0xFE) == -448.0
    assert rf.e4m3_value(0x08) == 2.0 ** -6             # smallest normal
    assert rf.e4m3_value(0x01) == 2.0 ** -9             # smallest subnormal
    assert rf.e4m3_value(0x07) == 7 * 2.0 ** -9         # largest subnormal
    assert rf.e4m3_value(0x38) == 1.0 and rf.e4m3_value(0x40) == 2.0
    assert rf.e4m3_value(0x39) == 1.125                 # one mantissa step above 1
    assert rf.e4m3_value(0xB8) == -1.0
    assert math.isnan(rf.e4m3_value(0x7F)) and math.isnan(rf.e4m3_value(0xFF))
    finite = [c for c in range(256) if not math.isnan(rf.e4m3_value(c))]
    assert len(finite) == 254
    pos = [rf.e4m3_value(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))     # codes 0..126 increase


def test_e4m3_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if not math.isnan(rf.e4m3_value(c))], dtype=np.uint8)
    vals = np.array([rf.e4m3_value(int(c)) for c in codes])
    vals[codes == 0x80] = -0.0
    assert np.array_equal(rf.e4m3_round(vals), codes)
    assert np.array_equal(rf.e4m3_decode(codes), vals)


def test_e4m3_ties_go_to_the_even_code_and_large_values_saturate():
    pos = [rf.e4m3_value(c) for c in range(0x7F)]
    for c in range(0x7E):
        mid = 0.5 * (pos[c] + pos[c + 1])              # exact in float64
        even = c if c % 2 == 0 else c + 1
        assert rf.e4m3_round(np.array([mid]))[0] == even, c
        assert rf.e4m3_round(np.array([-mid]))[0] == (0x80 | even), c
        below = np.nextafter(mid, 0.0)
        above = np.nextafter(mid, np.inf)
        assert rf.e4m3_round(np.array([below]))[0] == c
        assert rf.e4m3_round(np.array([above]))[0] == c + 1
    assert list(rf.e4m3_round(np.array([448.0, 460.0, 1e30, -1e30]))) == [0x7E, 0x7E, 0x7E, 0xFE]


def test_e4m3_round_matches_an_independent_conversion():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(20000) * 2.0 ** -7,
                        rng.uniform(-448, 448, 20000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(rf.e4m3_round(x), ref)


def test_block_quantization_scale_and_error_bound():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((128, 64)) * 3).astype(np.float32)
    codes, scale = rf.quantize_block_e4m3(x)
    amax = np.max(np.abs(x))
    assert scale == np.float32(amax / np.float32(448))
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert codes[i] & 0x7F == 0x7E                      # the largest element maps to +-448
    deq = rf.e4m3_decode(codes) * np.float64(scale)
    err = np.abs(deq - x)
    normal = np.abs(x) * (448.0 / amax) >= 2.0 ** -6
    # half a mantissa step (2^-4 relative) plus the float32 rounding of the scaling
    assert np.all(err[normal] <= np.abs(x[normal]) * (2.0 ** -4 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * scale * (1 + 1e-6))
    zeros, one = rf.quantize_block_e4m3(np.zeros((3, 8), dtype=np.float32))
    assert one == 1.0 and not zeros.any()


def test_problem_quantization_covers_partial_prefix_block():
    p = rf.make_problem("BNSD", 1, [(100, 8, 16, 32)], 2, 2, 64, 0.8)   # Lp = 100: partial block
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 2, p.geoms[0].length, 64)).astype(np.float32)
    codes, scales = rf.quantize_e4m3(p, x, 2)
    assert scales.shape == (2, p.t_qblk)
    # the partial block's scale comes from its 100 valid rows only
    assert scales[1, 0] == np.float32(np.max(np.abs(x[0, 1, :100])) / np.float32(448))
    deq = rf.dequantize_e4m3(p, codes, scales, 2)
    assert np.max(np.abs(deq - x)) <= np.max(np.abs(x)) * 2.0 ** -4


# ---------------- precision "fp8" (reading R24): V on power-of-two scales ----------------

def test_pow2_exponent_is_the_smallest_fitting_integer():
    rng = np.random.default_rng(6)
    vals = list(rng.lognormal(0.0, 4.0, 500)) + [448.0 * 2.0 ** k for k in range(-20, 20)]
    vals += [float(np.nextafter(448.0 * 2.0 ** k, np.inf)) for k in range(-10, 10)]
    vals += [float(np.nextafter(448.0 * 2.0 ** k, 0.0)) for k in range(-10, 10)]
    for a in vals:
        brute = next(e for e in range(-200, 200) if a <= 448.0 * 2.0 ** e)   # scan from below
        assert rf.pow2_exponent(a) == brute, a
    assert rf.pow2_exponent(0.0) == 0


def test_pow2_block_quantization_matches_an_independent_conversion():
    rng = np.random.default_rng(7)
    for scale in (3.0, 0.01, 500.0):
        x = (rng.standard_normal((128, 128)) * scale).astype(np.float32)
        codes, e = rf.quantize_block_e4m3_pow2(x)
        amax = float(np.max(np.abs(x)))
        assert amax <= 448.0 * 2.0 ** e and amax > 448.0 * 2.0 ** (e - 1)
        # the scaling by 2^-e is exact, so a library cast of the scaled values must agree
        ref = torch.from_numpy((x.astype(np.float64) * 2.0 ** -e).astype(np.float32)) \
            .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes, ref)
        top = rf.e4m3_decode(codes[np.unravel_index(np.argmax(np.abs(x)), x.shape)])
        assert 224.0 <= abs(top) <= 448.0                   # the largest value lands in the top binade
        deq = rf.e4m3_decode(codes) * 2.0 ** e
        err = np.abs(deq - x)
        normal = np.abs(x) * 2.0 ** -e >= 2.0 ** -6
        assert np.all(err[normal] <= np.abs(x[normal]) * 2.0 ** -4)
        assert np.all(err[~normal] <= 2.0 ** -10 * 2.0 ** e)
    zeros, e0 = rf.quantize_block_e4m3_pow2(np.zeros((4, 8), dtype=np.float32))
    assert e0 == -127 and not zeros.any()              # never the row's largest exponent


def test_fp8_v_quantization_covers_partial_prefix_block():
    p = rf.make_problem("TND", 1, [(100, 8, 16, 32), (0, 8, 16, 16)], 4, 2, 128, 0.8)
    rng = np.random.default_rng(8)
    t_rows = sum(g.length for g in p.geoms)
    x = rng.standard_normal((t_rows, 2, 128)).astype(np.float32)
    codes, exps = rf.quantize_v_fp8(p, x, 2)
    assert exps.shape == (2, p.t_qblk) and exps.dtype == np.int32
    # the partial prefix block (Lp = 100) takes its exponent from its 100 valid rows
    assert exps[1, 0] == rf.pow2_exponent(float(np.max(np.abs(x[:100, 1]))))
    deq = rf.dequantize_v_fp8(p, codes, exps, 2)
    assert np.max(np.abs(deq - x)) <= np.max(np.abs(x)) * 2.0 ** -4


def test_fp8_probability_bound_holds_for_explicitly_rounded_probabilities():
    """Round every probability to E4M3 by hand (on a power-of-two scale that keeps them in
    the normal range) and check the output change against the oracle's bound."""
    w = dict(layout="BNSD", batch=1, seqs=[(64, 8, 16, 32)], n1=2, n2=2, d=64, sparsity=0.8)
    p = rf.make_problem(w["layout"], 1, w["seqs"], 2, 2, 64, 0.8)
    rng = np.random.default_rng(9)
    L = p.geoms[0].length
    q, k, v = (rng.standard_normal((1, 2, L, 64)) * 0.8 for _ in range(3))
    qb, kb = rf.pooled_means(p, q, 2), rf.pooled_means(p, k, 2)
    idx, num = rf.select(p, qb, kb)
    items = [(t, n) for t in (0, 3, 10, 20) for n in (0, 1)]
    exact = rf.attention(p, q, k, v, idx, num, 0.125, items)
    bound = rf.fp8_probability_error_bound(p, q, k, v, idx, num, 0.125, items)
    table = rf.qblock_table(p)
    for (t, n) in items:
        s, g, b = table[t]
        rows = rf.block_rows(g, b)
        keys = [r for j in idx[t, n, :num[t, n]] for r in rf.block_rows(g, int(j))]
        lg = 0.125 * (q[0, n, rows.start:rows.stop] @ k[0, n, keys].T)
        lg -= lg.max(axis=1, keepdims=True)
        pr = np.exp(lg)
        # on 2^6 the largest probability (1) sits at 64: values down to 2^-12 stay normal
        keep = pr >= 2.0 ** -12
        pq = np.where(keep, rf.e4m3_decode(rf.e4m3_round(pr * 64.0)) / 64.0, pr)
        o_round = (pq @ v[0, n, keys]) / pr.sum(axis=1, keepdims=True)
        assert np.all(np.abs(o_round - exact[(t, n)]) <= bound[(t, n)] + 1e-12)


@pytest.mark.parametrize("u", [0, 3, 8])
def test_fp8_probability_bound_covers_block_shifts_and_subnormals(u):
    """Round P * 2^u * 2^(e_j - e_max) to E4M3 exactly as the reading states, with V
    exponents that differ between blocks (so small probabilities of low-exponent blocks
    fall below the normal range), and check the change against the bound."""
    p = rf.make_problem("BNSD", 1, [(64, 8, 16, 32)], 2, 2, 64, 0.8)
    rng = np.random.default_rng(10 + u)
    L = p.geoms[0].length
    q, k = (rng.standard_normal((1, 2, L, 64)) * 1.5 for _ in range(2))
    v = rng.standard_normal((1, 2, L, 64))
    qb, kb = rf.pooled_means(p, q, 2), rf.pooled_means(p, k, 2)
    idx, num = rf.select(p, qb, kb)
    vexp = rng.integers(-9, -2, size=(2, p.t_qblk)).astype(np.int32)
    items = [(t, n) for t in (0, 2, 9, 25) for n in (0, 1)]
    exact = rf.attention(p, q, k, v, idx, num, 0.125, items)
    bound = rf.fp8_probability_error_bound(p, q, k, v, idx, num, 0.125, items, v_exps=vexp)
    table = rf.qblock_table(p)
    for (t, n) in items:
        s, g, b = table[t]
        rows = rf.block_rows(g, b)
        blocks = [int(j) for j in idx[t, n, :num[t, n]]]
        keys = [r for j in blocks for r in rf.block_rows(g, j)]
        e = np.concatenate([np.full(len(rf.block_rows(g, j)), vexp[n, t - b + j]) for j in blocks])
        lg = 0.125 * (q[0, n, rows.start:rows.stop] @ k[0, n, keys].T)
        lg -= lg.max(axis=1, keepdims=True)
        pr = np.exp(lg)
        f = 2.0 ** (u + e - e.max())[None, :]
        pq = rf.e4m3_decode(rf.e4m3_round(pr * f)) / f
        o_round = (pq @ v[0, n, keys]) / pr.sum(axis=1, keepdims=True)
        assert np.all(np.abs(o_round - exact[(t, n)]) <= bound[(t, n)] + 1e-12)
