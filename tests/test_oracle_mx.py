"""Pins for the oracle's MXFP4 attention (UOS scaling, PNQ; CPU only).

E2M1 is fixed by its bit layout; the pins check the table in closed form, every
rounding midpoint, saturation and an independent conversion (ml_dtypes'
float4_e2m1fn, which the oracle does not use).  UOS is pinned by its defining
inequality and boundary, PNQ by the exact normalization it guarantees, the
integer-reference reading by its invariance, the whole query-block function by
a pure-Python element loop on a tiny case, and the key grouping by a hand-built
example with a partial prefix block.
"""
import math

import ml_dtypes
import numpy as np
import pytest

from oracle import mxattention as mx
from oracle import rainfusion as rfo

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_table_in_closed_form():
    assert [mx.e2m1_value(c) for c in range(8)] == GRID
    assert [mx.e2m1_value(c | 8) for c in range(8)] == [-v for v in GRID]
    assert mx.E2M1_MAX == 6.0 and mx.MX_BLOCK == 32 and mx.QMAX_UOS == 7.25


def test_e2m1_grid_points_are_fixed_and_midpoints_go_to_the_even_code():
    codes = mx.e2m1_round_codes(np.array(GRID))
    assert list(codes) == list(range(8))
    for c in range(7):
        mid = 0.5 * (GRID[c] + GRID[c + 1])
        even = c if c % 2 == 0 else c + 1
        assert mx.e2m1_round_codes(np.array([mid]))[0] == even, mid
        assert mx.e2m1_round_codes(np.array([-mid]))[0] == (8 | even), mid
        assert mx.e2m1_round_codes(np.array([np.nextafter(mid, 0.0)]))[0] == c
        assert mx.e2m1_round_codes(np.array([np.nextafter(mid, 9.0)]))[0] == c + 1
    # 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4; beyond 6 saturates
    vals = mx.e2m1_decode(mx.e2m1_round_codes(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.25, 1e9])))
    assert list(vals) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 6.0]


def test_e2m1_matches_an_independent_conversion():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-6, 6, 50000), rng.standard_normal(20000) * 0.4]).astype(np.float32)
    ref = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = mx.e2m1_decode(mx.e2m1_round_codes(x))
    assert np.array_equal(np.abs(got), np.abs(ref))
    nz = ref != 0
    assert np.array_equal(np.sign(got[nz]), np.sign(ref[nz]))


def test_uos_exponent_bound_and_boundary():
    rng = np.random.default_rng(5)
    for amax in np.exp(rng.uniform(-60, 60, 5000)):
        e = mx.uos_exponent(float(amax))
        r = amax / 2.0 ** e
        assert 7.25 / 2 < r <= 7.25, (amax, e)
    for k in range(-30, 31):
        b = 7.25 * 2.0 ** k
        assert mx.uos_exponent(b) == k                       # at the boundary: no clipping headroom lost
        assert mx.uos_exponent(float(np.nextafter(b, np.inf))) == k + 1
        assert mx.uos_exponent(float(np.nextafter(b, 0.0))) == k
    assert mx.uos_exponent(0.0) == 0


def test_ocp_exponent_bound():
    rng = np.random.default_rng(6)
    for amax in np.exp(rng.uniform(-60, 60, 5000)):
        e = mx.ocp_exponent(float(amax))
        assert 4.0 <= amax / 2.0 ** e < 8.0
    assert mx.ocp_exponent(1.0) == -2 and mx.ocp_exponent(6.0) == 0 and mx.ocp_exponent(8.0) == 1


def test_group_quantization_keeps_grid_values_and_scales_by_powers_of_two():
    g = np.array([6.0, 1.5, 0.5, 3.0, -4.0, 0.0, 2.0, -1.0]) * 2.0 ** -3   # amax 0.75 -> e = -3
    assert np.array_equal(mx.quantize_group(g), g)
    rng = np.random.default_rng(8)
    x = rng.standard_normal(32)
    for k in (-9, -1, 0, 4, 17):
        assert np.array_equal(mx.quantize_group(x * 2.0 ** k), mx.quantize_group(x) * 2.0 ** k)
    # a group is at most 32 wide: a large value elsewhere does not change this group
    row = rng.standard_normal(64)
    row2 = row.copy()
    row2[40] = 1e6
    assert np.array_equal(mx.quantize_rows(row[None])[0, :32], mx.quantize_rows(row2[None])[0, :32])


def test_uos_error_is_below_ocp_on_gaussian_groups():
    # [MX] abstract: UOS improves on the OCP scale choice; on Gaussian data its
    # mean squared error is lower.
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4000, 32))
    e_uos = np.mean([(mx.quantize_group(r, "uos") - r) ** 2 for r in x])
    e_ocp = np.mean([(mx.quantize_group(r, "ocp") - r) ** 2 for r in x])
    assert e_uos < e_ocp


def _geom():
    # P = 100 text rows, one 16 x 16 frame: 256 aligned tokens = 2 video blocks, nothing
    # promoted, one partial prefix block of 100 rows.
    return rfo.geometry(100, 1, 16, 16, 0.5)


def test_key_groups_follow_block_boundaries():
    g = _geom()
    assert (g.lp, g.n_pb, g.nb) == (100, 1, 2)
    assert [(r.start, r.stop) for r in mx.key_groups(g, 0)] == [(0, 32), (32, 64), (64, 96), (96, 100)]
    assert [(r.start, r.stop) for r in mx.key_groups(g, 1)] == [(100, 132), (132, 164), (164, 196), (196, 228)]
    assert [(r.start, r.stop) for r in mx.key_groups(g, 2)] == [(228, 260), (260, 292), (292, 324), (324, 356)]


def test_v_groups_do_not_cross_the_prefix_end():
    g = _geom()
    rng = np.random.default_rng(2)
    v = rng.standard_normal((g.length, 8))
    base = mx.quantize_v(v, g)
    v2 = v.copy()
    v2[100, :] = 1e5           # first row of the first video block
    q2 = mx.quantize_v(v2, g)
    assert np.array_equal(base[:100], q2[:100])          # the 4-row prefix group 96..99 is untouched
    assert np.array_equal(base[132:], q2[132:])
    assert not np.array_equal(base[101:132], q2[101:132])


def _inputs(g, d, seed):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((g.length, d)) for _ in range(3))
    return mx.quantize_rows(q), mx.quantize_rows(k), mx.quantize_v(v, g)


def test_pnq_weights_sum_to_one_exactly():
    g = _geom()
    qq, kq, _ = _inputs(g, 64, 1)
    ones = np.ones((g.length, 64))
    for qb, keys in ((0, [0, 1, 2]), (2, [0, 2])):
        o = mx.attend_query_block_mx(qq, kq, ones, g, qb, keys, 0.125)
        assert np.max(np.abs(o - 1.0)) < 1e-14


def test_integer_reference_shift_does_not_change_the_output():
    g = _geom()
    qq, kq, vq = _inputs(g, 64, 3)
    ref = mx.attend_query_block_mx(qq, kq, vq, g, 1, [0, 1, 2], 0.3)
    for shift in (-7, -1, 2, 11):
        o = mx.attend_query_block_mx(qq, kq, vq, g, 1, [0, 1, 2], 0.3, m_shift=shift)
        assert np.max(np.abs(o - ref)) < 1e-12, shift


def test_without_p_quantization_it_is_the_plain_softmax_attention():
    g = _geom()
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((g.length, 64)) for _ in range(3))
    for qb, keys in ((0, [0, 1, 2]), (1, [0, 2]), (2, [0, 1, -1])):
        a = mx.attend_query_block_mx(q, k, v, g, qb, keys, 0.125, quantize_p=False)
        b = rfo.attend_query_block(q, k, v, g, qb, keys, 0.125)
        assert np.max(np.abs(a - b)) < 1e-12


def _brute_q(vals):
    """Group quantization by scanning: the smallest e with amax / 2^e <= 7.25, then each
    value to the nearest of +-GRID * 2^e, ties to the even grid index."""
    amax = max(abs(x) for x in vals)
    if amax == 0:
        return [0.0 for _ in vals]
    e = -300
    while amax / 2.0 ** e > 7.25:
        e += 1
    out = []
    for x in vals:
        y = min(abs(x) / 2.0 ** e, 6.0)
        best = 0
        for i in range(1, 8):
            d_new, d_best = abs(GRID[i] - y), abs(GRID[best] - y)
            if d_new < d_best or (d_new == d_best and i % 2 == 0):
                best = i
        out.append(math.copysign(GRID[best] * 2.0 ** e, x) if best else 0.0)
    return out


def test_query_block_against_an_element_loop():
    g = rfo.geometry(40, 1, 16, 16, 0.5)          # Lp = 40: a 40-row partial prefix block
    d = 32
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((g.length, d)) * 1.5 for _ in range(3))
    scale = 0.2
    qq = np.array([_brute_q(list(r)) for r in q])
    kq = np.array([_brute_q(list(r)) for r in k])
    vq = np.zeros_like(v)
    for b in range(g.n_blocks):
        for grp in mx.key_groups(g, b):
            for c in range(d):
                vq[grp.start:grp.stop, c] = _brute_q(list(v[grp.start:grp.stop, c]))
    assert np.array_equal(qq, mx.quantize_rows(q)) and np.array_equal(vq, mx.quantize_v(v, g))
    qb, keys = 2, [0, 2]
    got = mx.attend_query_block_mx(qq, kq, vq, g, qb, keys, scale)
    groups = [grp for b in keys for grp in mx.key_groups(g, b)]
    for i, qi in enumerate(rfo.block_rows(g, qb)):
        xs = {j: scale * sum(qq[qi, c] * kq[j, c] for c in range(d)) / math.log(2.0)
              for grp in groups for j in grp}
        m = math.ceil(max(xs.values()))
        pq = {}
        for grp in groups:
            vals = _brute_q([2.0 ** (xs[j] - m) for j in grp])
            pq.update(zip(grp, vals))
        l = sum(pq.values())
        for c in range(d):
            o = sum(pq[j] * vq[j, c] for j in pq) / l
            assert abs(o - got[i, c]) < 1e-12, (i, c)


def test_mx_attention_is_close_to_the_exact_attention():
    g = _geom()
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((g.length, 128)) for _ in range(3))
    qq, kq, vq = mx.quantize_rows(q), mx.quantize_rows(k), mx.quantize_v(v, g)
    a = mx.attend_query_block_mx(qq, kq, vq, g, 1, [0, 1, 2], 128 ** -0.5)
    b = rfo.attend_query_block(q, k, v, g, 1, [0, 1, 2], 128 ** -0.5)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0.01 < rel < 0.25, rel        # FP4 is coarse, but the output stays close


def test_vectorized_exponents_equal_the_scalar_rule():
    rng = np.random.default_rng(13)
    a = np.concatenate([np.exp(rng.uniform(-80, 80, 3000)), 7.25 * 2.0 ** np.arange(-40, 40),
                        np.nextafter(7.25 * 2.0 ** np.arange(-40, 40), np.inf), [0.0]])
    assert list(mx.uos_exponents(a)) == [mx.uos_exponent(float(x)) for x in a]


def test_vectorized_rows_and_columns_equal_group_by_group_rounding():
    g = rfo.geometry(77, 2, 17, 33, 0.8)          # partial prefix block, ragged grid
    rng = np.random.default_rng(14)
    x = rng.standard_normal((g.length, 64)) * np.exp(rng.uniform(-3, 3, (g.length, 1)))
    rows = mx.quantize_rows(x)
    for r in range(0, g.length, 37):
        for c0 in (0, 32):
            assert np.array_equal(rows[r, c0:c0 + 32], mx.quantize_group(x[r, c0:c0 + 32]))
    cols = mx.quantize_v(x, g)
    for b in range(g.n_blocks):
        for grp in mx.key_groups(g, b):
            for d in (0, 5, 63):
                assert np.array_equal(cols[grp.start:grp.stop, d], mx.quantize_group(x[grp.start:grp.stop, d]))
