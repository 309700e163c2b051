"""Pins of the oracle's element codecs and scale rules against things other than itself:
library decoders (ml_dtypes, torch), exact rational arithmetic, brute force and hand values."""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# OCP MX v1.0 E2M1 magnitudes for codes 0..7 (the format definition; the pages only name E2M1).
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_all_codes(orc):
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        v = orc.e2m1_value(c)
        expect = E2M1_MAGNITUDES[c & 7] * (-1.0 if c & 8 else 1.0)
        assert v == expect and math.copysign(1, v) == math.copysign(1, expect), c
        assert v == lib_vals[c]


def _e2m1_probe_values():
    rng = np.random.default_rng(0)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    pts = [ties, np.nextafter(ties, 0), np.nextafter(ties, 10),
           np.array(E2M1_MAGNITUDES, dtype=np.float32), np.array([6.0, 6.5, 7.0, 7.99, 8.0, 1e30], np.float32),
           np.array([1e-30, 1e-45, 0.1, 0.2499], np.float32),
           rng.uniform(-8, 8, 20000).astype(np.float32), rng.standard_normal(5000).astype(np.float32) * 3]
    v = np.concatenate(pts)
    return np.concatenate([v, -v, np.array([0.0, -0.0], np.float32)])


def test_e2m1_encode_matches_library_and_bruteforce(orc):
    vals = _e2m1_probe_values()
    lib_codes = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    grid = np.array(E2M1_MAGNITUDES)
    for v, lc in zip(vals.tolist(), lib_codes.tolist()):
        c = orc.e2m1_encode(v)
        assert c == lc, (v, c, lc)
        # brute force: nearest magnitude, ties to the even code, saturating at 6, sign kept
        a = min(abs(v), 6.0)
        d = np.abs(grid - a)
        best = np.flatnonzero(d == d.min())
        mag = int(best[0] if best.size == 1 else [b for b in best if b % 2 == 0][0])
        assert c == (mag | (8 if math.copysign(1, v) < 0 else 0)), v


def test_e2m1_tie_table(orc):
    # ties go to the even code: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2.0, 2.5->2.0, 3.5->4.0, 5->4.0
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in expect.items():
        assert orc.e2m1_encode(v) == c
        assert orc.e2m1_encode(-v) == c | 8
    assert orc.e2m1_encode(-0.1) == 0x8  # negative values rounding to zero keep the sign


def test_e4m3_decode_all_codes(orc):
    lib_vals = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tv = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = orc.e4m3_value(c)
        if math.isnan(lib_vals[c]):
            assert math.isnan(v) and c & 0x7F == 0x7F
        else:
            assert v == lib_vals[c] == tv[c], c
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_in_range_matches_libraries(orc):
    finite = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    finite = np.unique(np.abs(finite[~np.isnan(finite)]))
    mids = (finite[1:] + finite[:-1]) / 2
    rng = np.random.default_rng(1)
    v = np.concatenate([finite, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.uniform(0, 464, 20000), np.exp(rng.uniform(-16, 6, 20000))]).astype(np.float32)
    v = v[v <= 464.0]
    v = np.concatenate([v, -v])
    lib_codes = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    t_codes = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, lc, tc in zip(v.tolist(), lib_codes.tolist(), t_codes.tolist()):
        c = orc.e4m3_encode(x)
        assert c == lc == tc, (x, c, lc, tc)


def test_e4m3_encode_saturates(orc):
    for x in [464.0001, 480.0, 500.0, 1e6, 3.0e38, float("inf")]:
        assert orc.e4m3_encode(x) == 0x7E
        assert orc.e4m3_encode(-x) == 0xFE


def test_e8m0_decode_all_codes(orc):
    lib_vals = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    for c in range(256):
        v = orc.e8m0_value(c)
        if c == 255:
            assert math.isnan(v) and math.isnan(lib_vals[c])
        else:
            assert v == lib_vals[c] == 2.0 ** (c - 127)


def _bf16_positive_finite():
    bits = np.arange(1, 0x7F80, dtype=np.uint32)  # exponent field 0..254, every mantissa, no zero
    return (bits << 16).view(np.float32).astype(np.float64)


def _exact_exponent(amax, elem_emax, elem_max, rule):
    """Integer arithmetic on the exact rational value of amax."""
    if amax == 0:
        return -127
    fr = Fraction(amax)
    # floor(log2 fr): largest E with 2^E <= fr
    E = fr.numerator.bit_length() - fr.denominator.bit_length()
    while Fraction(2) ** E > fr:
        E -= 1
    while Fraction(2) ** (E + 1) <= fr:
        E += 1
    if rule == "even":
        e = E - elem_emax
    else:
        e = E - 64
        while fr > elem_max * Fraction(2) ** e:
            e += 1
    return max(-127, min(127, e))


@pytest.mark.parametrize("fmt,elem_emax,elem_max", [("mxfp4", 2, 6), ("mxfp8", 8, 448)])
@pytest.mark.parametrize("rule", ["even", "ceil"])
def test_mx_exponent_exhaustive_over_bf16(orc, fmt, elem_emax, elem_max, rule):
    f = orc.MXFP4 if fmt == "mxfp4" else orc.MXFP8
    r = orc.EVEN if rule == "even" else orc.CEIL
    vals = _bf16_positive_finite()
    # exact rational definition on a stride through all 32,639 values plus every binade edge
    check = np.unique(np.concatenate([vals[::7], vals[:300], vals[-300:]]))
    for a in check.tolist():
        assert orc.mx_exponent(a, f, r) == _exact_exponent(a, elem_emax, elem_max, rule), a
    # all values: closed form on the exponent/mantissa fields (m in [1,2), amax = m * 2^E)
    m, E = np.frexp(vals)
    m, E = m * 2, E - 1
    if rule == "even":
        expect = E - elem_emax
    else:
        expect = E - elem_emax + (m > (1.5 if fmt == "mxfp4" else 1.75))
    expect = np.clip(expect, -127, 127)
    got = np.array([orc.mx_exponent(a, f, r) for a in vals.tolist()])
    assert np.array_equal(got, expect)


def test_mx_exponent_golden(orc):
    n = 0
    with open(os.path.join(GOLDEN, "scale_exponents.txt")) as fh:
        for line in fh:
            if not line.strip() or line.startswith("#"):
                continue
            amax, fmt, rule, e = line.split()
            f = orc.MXFP4 if fmt == "mxfp4" else orc.MXFP8
            r = orc.EVEN if rule == "even" else orc.CEIL
            assert orc.mx_exponent(float(amax), f, r) == int(e), line
            n += 1
    assert n >= 20


def test_mx_exponent_clamp(orc):
    # bf16 subnormal amax: floor(log2) = -133 -> e clamps at -127 under both rules
    for a in [2.0 ** -133, 2.0 ** -126, 2.0 ** -125 * 1.25]:
        assert orc.mx_exponent(a, orc.MXFP4, orc.EVEN) == -127
        assert orc.mx_exponent(a, orc.MXFP4, orc.CEIL) == -127
    # 1.75 * 2^-125: EVEN -127, CEIL -125 - 2 + 1 = -126 (just above the clamp)
    assert orc.mx_exponent(2.0 ** -125 * 1.75, orc.MXFP4, orc.EVEN) == -127
    assert orc.mx_exponent(2.0 ** -125 * 1.75, orc.MXFP4, orc.CEIL) == -126
    assert orc.mx_exponent(2.0 ** -120, orc.MXFP4, orc.EVEN) == -122
    assert orc.mx_exponent(2.0 ** -120, orc.MXFP4, orc.CEIL) == -122
    big = float(np.float32(3.3895314e38))  # largest bf16
    assert orc.mx_exponent(big, orc.MXFP4, orc.EVEN) == 125
    assert orc.mx_exponent(big, orc.MXFP4, orc.CEIL) == 126


def test_bf16_value(orc):
    for bits, v in [(0x3F80, 1.0), (0xBF80, -1.0), (0x0001, 2.0 ** -133), (0x7F7F, 3.3895313892515355e38),
                    (0x4040, 3.0)]:
        assert orc.bf16_value(bits) == v
