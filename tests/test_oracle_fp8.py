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
