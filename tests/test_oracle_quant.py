"""Pins of the oracle's block quantizers, dequantizer, scale layout and GEMM.

Each check is chosen so that a plausible slip in the oracle (wrong rule, dropped sign, swapped
nibbles, wrong block index, transposed operand, missing global scale) fails at least one test:
  - MX quantize against a construction from library casts (ml_dtypes) and exact exponents;
  - NVFP4 against numpy fp32 arithmetic plus ml_dtypes casts, a hand-worked block, and its
    order-free definition in exact rational arithmetic (nearest E4M3 scale to amax / (6 g),
    nearest E2M1 value to x / (dec(s) g)) wherever no rounding midpoint is within reach of the
    fp32 steps;
  - invariants: all-zero blocks, saturation, idempotence, value bounds;
  - scale layout: bijection, round trip, hand-worked offsets;
  - GEMM: numpy fp64 matmul of library-decoded operands, exact integer products, selection.
"""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_mx_b200 import synth


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _exp_exact(amax, elem_emax, elem_max, rule):
    if amax == 0:
        return -127
    m, E = math.frexp(amax)
    E -= 1
    if rule == "even":
        e = E - elem_emax
    else:
        e = E - elem_emax - 1
        while amax > math.ldexp(elem_max, e):
            e += 1
    return max(-127, min(127, e))


def _mx_reference(x, fmt, rule):
    """Library-cast construction: x * 2^-e cast by ml_dtypes (RNE), saturating."""
    xf = x.float().numpy().astype(np.float64)
    rows, K = xf.shape
    blocks = xf.reshape(rows, K // 32, 32)
    amax = np.abs(blocks).max(-1)
    emax, emaxval = (8, 448.0) if fmt == "mxfp8" else (2, 6.0)
    e = np.vectorize(lambda a: _exp_exact(a, emax, emaxval, rule))(amax).astype(np.int64)
    v = np.ldexp(blocks, -e[..., None])
    if fmt == "mxfp8":
        codes = np.clip(v, -448, 448).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    else:
        codes = v.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    return codes.reshape(rows, K), (e + 127).astype(np.uint8)


def _unpack_fp4(q):
    lo, hi = q & 0xF, q >> 4
    return np.stack([lo, hi], -1).reshape(q.shape[0], -1)


def _adversarial_bf16(rows, K, seed, huge=3.0e38, bs=32):
    """Random rows plus blocks built to sit on ties, zeros, saturation and tiny amax."""
    g = np.random.default_rng(seed)
    x = g.standard_normal((rows, K)).astype(np.float32) * np.exp(g.uniform(-6, 6, (rows, 1))).astype(np.float32)
    blocks = x.reshape(-1, bs)
    nb = blocks.shape[0]
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    for b in range(0, nb, 7):
        kind = (b // 7) % 6
        if kind == 0:
            blocks[b] = 0.0
        elif kind == 1:  # scaled ties with amax exactly 6 * 2^k
            k = g.integers(-20, 20)
            blocks[b] = np.ldexp(g.choice(ties, bs) * g.choice([-1, 1], bs), k)
            blocks[b, 0] = np.ldexp(6.0, k)
        elif kind == 2:  # saturation under EVEN: amax = 7.5 * 2^k
            k = g.integers(-10, 10)
            blocks[b, :] = np.ldexp(g.uniform(-7.5, 7.5, bs), k)
            blocks[b, 3] = np.ldexp(7.5, k)
        elif kind == 3:  # tiny amax near the -127 clamp
            blocks[b] = np.ldexp(g.uniform(-1, 1, bs), -128).astype(np.float32)
        elif kind == 4:  # negative zeros mixed with zeros
            blocks[b] = -0.0
            blocks[b, ::2] = 0.0
        else:  # one huge outlier
            blocks[b, 5] = huge
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", ["mxfp4", "mxfp8"])
@pytest.mark.parametrize("rule", ["even", "ceil"])
def test_mx_quantize_matches_library_construction(orc, fmt, rule):
    f = orc.MXFP4 if fmt == "mxfp4" else orc.MXFP8
    r = orc.EVEN if rule == "even" else orc.CEIL
    for seed, (rows, K) in enumerate([(5, 64), (37, 320), (64, 1024)]):
        x = _adversarial_bf16(rows, K, seed)
        q, sf = orc.quantize(x, f, r)
        codes_ref, sf_ref = _mx_reference(x, fmt, rule)
        assert np.array_equal(sf, sf_ref)
        codes = q if fmt == "mxfp8" else _unpack_fp4(q)
        assert np.array_equal(codes, codes_ref)


def test_fp4_nibble_order(orc):
    # element 2i -> low nibble, 2i+1 -> high nibble (OCP / torch float4_e2m1fn_x2 convention)
    x = torch.zeros(1, 32, dtype=torch.bfloat16)
    x[0, 0], x[0, 1], x[0, 2] = 6.0, -1.0, 0.5  # amax 6 -> e = 0 under both rules
    q, sf = orc.quantize(x, orc.MXFP4, orc.CEIL)
    assert sf[0, 0] == 127
    assert q[0, 0] == (0x7 | (0xA << 4))
    assert q[0, 1] == 0x1


def test_zero_blocks(orc):
    x = torch.zeros(3, 64, dtype=torch.bfloat16)
    x[1, 32:] = -0.0
    for f, r in [(orc.MXFP4, orc.EVEN), (orc.MXFP4, orc.CEIL), (orc.MXFP8, orc.EVEN), (orc.NVFP4, 0)]:
        q, sf = orc.quantize(x, f, r, g=1.0)
        assert np.all(sf == 0)
        if f == orc.MXFP8:
            assert np.all(q[1, 32:] == 0x80) and np.all(q[0] == 0)
        else:
            assert np.all(q[1, 16:] == 0x88) and np.all(q[0] == 0)


def test_even_rule_saturates(orc):
    for k in [-5, 0, 7]:
        x = torch.zeros(1, 32, dtype=torch.bfloat16)
        x[0, 4] = math.ldexp(7.5, k)
        x[0, 5] = -math.ldexp(7.5, k)
        q, sf = orc.quantize(x, orc.MXFP4, orc.EVEN)
        assert sf[0, 0] == 127 + k
        assert q[0, 2] == (0x7 | (0xF << 4))  # 7.5 * 2^k / 2^k -> saturates to 6.0
        q, sf = orc.quantize(x, orc.MXFP4, orc.CEIL)  # CEIL never clips: amax/2^e <= 6
        assert sf[0, 0] == 127 + k + 1
        assert q[0, 2] == (0x6 | (0xE << 4))  # 7.5 * 2^k / 2^(k+1) = 3.75 -> 4.0 (code 6)


def _codes_max(q, K):
    return (_unpack_fp4(q) & 7).reshape(q.shape[0], K // 32, 32).max(-1)


@pytest.mark.parametrize("rule", ["even", "ceil"])
def test_idempotence(orc, rule):
    r = orc.EVEN if rule == "even" else orc.CEIL
    # (an outlier near the bf16 maximum is left out: CEIL can round it up past bf16's range)
    x = _adversarial_bf16(16, 512, 3, huge=3.0e30)
    q, sf = orc.quantize(x, orc.MXFP4, r)
    d = orc.dequantize(q, sf, 512, orc.MXFP4)
    xd = torch.from_numpy(d).to(torch.bfloat16)
    assert np.array_equal(xd.double().numpy(), d)  # dequantized values are exact in bf16 here
    q2, sf2 = orc.quantize(xd, orc.MXFP4, r)
    d2 = orc.dequantize(q2, sf2, 512, orc.MXFP4)
    assert np.array_equal(d, d2)  # value idempotence for both rules
    cmax = _codes_max(q, 512).reshape(-1)
    same = (_unpack_fp4(q).reshape(-1, 32) == _unpack_fp4(q2).reshape(-1, 32)).all(-1)
    if rule == "even":
        assert same.all()
    else:
        assert same[cmax >= 6].all()  # max value 4 or 6 keeps e; max value 3 re-quantizes one binade lower
    q3, sf3 = orc.quantize(torch.from_numpy(d2).to(torch.bfloat16), orc.MXFP4, r)
    assert np.array_equal(q3, q2) and np.array_equal(sf3, sf2)  # fixed point after one pass


def test_ceil_code3_block_changes_bytes_not_values(orc):
    # scaled amax 3.25 (in (3, 3.5)) has max code 3 (=3.0); re-quantizing picks e-1
    x = torch.zeros(1, 32, dtype=torch.bfloat16)
    x[0, 0] = 3.25 * 2.0
    x[0, 1] = 1.0
    q, sf = orc.quantize(x, orc.MXFP4, orc.CEIL)
    assert sf[0, 0] == 128 and (q[0, 0] & 0xF) == 5  # e = 1, 3.25 -> 3.0
    d = orc.dequantize(q, sf, 32, orc.MXFP4)
    q2, sf2 = orc.quantize(torch.from_numpy(d).to(torch.bfloat16), orc.MXFP4, orc.CEIL)
    assert sf2[0, 0] == 127 and (q2[0, 0] & 0xF) == 7
    assert np.array_equal(orc.dequantize(q2, sf2, 32, orc.MXFP4), d)


def _nvfp4_reference(x, g):
    """numpy fp32 IEEE steps + ml_dtypes casts."""
    xf = x.float().numpy()
    rows, K = xf.shape
    b = xf.reshape(rows, K // 16, 16)
    amax = np.abs(b).max(-1).astype(np.float32)
    g = np.float32(g)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):  # u saturates to 448 below
        u = (amax / np.float32(6.0)) / g
    s = np.minimum(u, np.float32(448.0)).astype(ml_dtypes.float8_e4m3fn)
    s = np.where(amax == 0, np.zeros_like(s), s)
    sdec = s.astype(np.float32)
    d = sdec * g
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):  # saturating products are intended
        rcp = np.float32(1.0) / d
        v = b * rcp[..., None]
    codes = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    zero = (d == 0)[..., None] & np.ones_like(codes, dtype=bool)
    codes = np.where(zero, np.where(np.signbit(b), 8, 0).astype(np.uint8), codes)
    return codes.reshape(rows, K), s.view(np.uint8)


def test_nvfp4_matches_fp32_library_construction(orc):
    for seed, (rows, K) in enumerate([(7, 48), (33, 256), (64, 1024)]):
        x = _adversarial_bf16(rows, K, 10 + seed, huge=3.0e6, bs=16)
        g, amax = orc.global_scale(x)
        assert g == np.float32(amax) / np.float32(2688.0)
        q, sf = orc.quantize(x, orc.NVFP4, 0, g=float(g))
        codes_ref, sf_ref = _nvfp4_reference(x, g)
        assert np.array_equal(sf, sf_ref)
        assert np.array_equal(_unpack_fp4(q), codes_ref)
        sdec = np.vectorize(orc.e4m3_value)(sf)
        assert np.all(sdec <= 448.0) and np.all(sdec >= 0)


def test_nvfp4_hand_block(orc):
    # g = 1/64; block amax = 6 g = 0.09375 -> u = 1 -> s = E4M3(1.0) = 0x38, d = g, v = x / g
    g = 1.0 / 64
    vals = [0.09375, -0.046875, 0.0234375, 0.0078125] + [0.0] * 12  # 6g, -3g, 1.5g, 0.5g
    x = torch.tensor([vals], dtype=torch.bfloat16)
    q, sf = orc.quantize(x, orc.NVFP4, 0, g=g)
    assert sf[0, 0] == 0x38
    assert q[0, 0] == (0x7 | (0xD << 4)) and q[0, 1] == (0x3 | (0x1 << 4))
    d = orc.dequantize(q, sf, 16, orc.NVFP4, g=g)
    assert np.allclose(d[0, :4], vals[:4], rtol=0, atol=0)


def test_nvfp4_reciprocal_overflow(orc):
    # g = 2^-140 is an fp32 subnormal.  A block with amax 1 has u = fl(fl(1/6) / g), far above 448,
    # so s saturates to 448 (0x7E) and d = 448 * 2^-140 = 1.75 * 2^-132, whose reciprocal overflows
    # fp32: r = +inf.  Then fl(x * r) is +-inf for every nonzero x (E2M1 saturates it to +-6, code 7
    # with the sign) and NaN for x = +-0, which encodes as a zero with x's sign.
    g = 2.0 ** -140
    d = np.float32(448.0) * np.float32(g)
    assert d == np.float32(1.75 * 2.0 ** -132)
    with np.errstate(over="ignore", divide="ignore"):
        assert np.isinf(np.float32(1.0) / d)
    tiny = float(torch.tensor(2.0 ** -133, dtype=torch.bfloat16))  # the smallest bf16 subnormal
    vals = [1.0, -1.0, 0.0, -0.0, tiny, -tiny, 0.5, -3.0] * 2
    x = torch.tensor([vals], dtype=torch.bfloat16)
    q, sf = orc.quantize(x, orc.NVFP4, 0, g=g)
    assert sf[0, 0] == 0x7E
    expect = [0x7, 0xF, 0x0, 0x8, 0x7, 0xF, 0x7, 0xF] * 2
    assert _unpack_fp4(q)[0].tolist() == expect
    # with g = 1/2688 the same block has d = 1/6 and r = 6: the tiny elements round to signed zeros
    q2, _ = orc.quantize(x, orc.NVFP4, 0, g=1.0 / 2688)
    assert _unpack_fp4(q2)[0, :6].tolist() == [0x7, 0xF, 0x0, 0x8, 0x0, 0x8]


def test_swizzle_layout(orc):
    for rows, kb in [(1, 1), (128, 4), (130, 5), (300, 160), (16, 8)]:
        total = orc.swizzled_bytes(rows, kb)
        assert total == ((rows + 127) // 128) * 128 * ((kb + 3) // 4) * 4
        offs = np.array([[orc.swizzle_offset(r, c, kb) for c in range(kb)] for r in range(rows)])
        assert len(np.unique(offs)) == rows * kb and offs.max() < total  # injective, in range
        sf = np.random.default_rng(rows).integers(1, 255, (rows, kb), dtype=np.uint8)
        sw = orc.swizzle(sf)
        assert np.array_equal(orc.unswizzle(sw, rows, kb), sf)
        mask = np.ones(total, bool)
        mask[offs.reshape(-1)] = False
        assert np.all(sw[mask] == 0)  # padding is zero
    # hand-worked offsets: tile (row-tile, col-tile) of 512 B, then (r%32)*16 + ((r%128)/32)*4 + c%4
    kb = 8  # two column tiles per row tile
    for (r, c), off in {(0, 0): 0, (0, 3): 3, (0, 4): 512, (1, 0): 16, (31, 0): 496, (32, 0): 4,
                        (96, 2): 14, (127, 7): 512 + 31 * 16 + 12 + 3, (128, 0): 1024,
                        (161, 5): 1024 + 512 + 16 + 4 + 1}.items():
        assert orc.swizzle_offset(r, c, kb) == off


def _lib_dequant(q, sf, K, fmt, g=1.0):
    if fmt == "mxfp8":
        el = q.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
        bs = 32
    else:
        el = _unpack_fp4(q).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
        bs = 16 if fmt == "nvfp4" else 32
    if fmt == "nvfp4":
        sc = sf.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * g
    else:
        sc = sf.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    return el * np.repeat(sc, bs, axis=1)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
def test_gemm_matches_numpy_fp64(orc, fmt):
    f = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4, "mxfp8": orc.MXFP8}[fmt]
    M, N, K = 9, 13, 192
    A = synth.random_bf16((M, K), 1)
    W = synth.random_bf16((N, K), 2, std=0.02)
    gA = gW = 1.0
    if fmt == "nvfp4":
        gA, _ = orc.global_scale(A)
        gW, _ = orc.global_scale(W)
    Aq, Asf = orc.quantize(A, f, orc.CEIL, g=float(gA))
    Wq, Wsf = orc.quantize(W, f, orc.EVEN, g=float(gW))
    out, absout = orc.gemm(Aq, Asf, Wq, Wsf, M, N, K, f, gA=float(gA), gB=float(gW))
    a = _lib_dequant(Aq, Asf, K, fmt, float(gA))
    b = _lib_dequant(Wq, Wsf, K, fmt, float(gW))
    ref = a @ b.T
    # fp64 summation order differs from numpy's: bound by a few ulps of sum |a b|
    assert np.all(np.abs(out - ref) <= 1e-13 * absout)
    assert np.allclose(absout, np.abs(a) @ np.abs(b).T, rtol=1e-12)
    assert np.array_equal(orc.dequantize(Aq, Asf, K, f, g=float(gA)), a)
    # selected rows / cols give the same entries
    rows, cols = np.array([8, 0, 3]), np.array([12, 5])
    sub, _ = orc.gemm(Aq, Asf, Wq, Wsf, M, N, K, f, gA=float(gA), gB=float(gW), rows=rows, cols=cols)
    assert np.array_equal(sub, out[np.ix_(rows, cols)])


def test_gemm_exact_integers(orc):
    # unit scales (E8M0 127) and E2M1 codes: 2*value is an integer, so the fp64 sum is exact
    rng = np.random.default_rng(5)
    M, N, K = 4, 6, 128
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    sfa = np.full((M, K // 32), 127, np.uint8)
    sfb = np.full((N, K // 32), 127, np.uint8)
    out, _ = orc.gemm(pack(ca), sfa, pack(cb), sfb, M, N, K, orc.MXFP4)
    twice = np.array([0, 1, 2, 3, 4, 6, 8, 12], np.int64)
    ia = twice[ca & 7] * np.where(ca & 8, -1, 1)
    ib = twice[cb & 7] * np.where(cb & 8, -1, 1)
    assert np.array_equal(out * 4, (ia @ ib.T).astype(np.float64))
    # a scale of 2^3 on one block of A row 0 multiplies exactly that block's contribution
    sfa2 = sfa.copy()
    sfa2[0, 1] = 130
    out2, _ = orc.gemm(pack(ca), sfa2, pack(cb), sfb, M, N, K, orc.MXFP4)
    part = (ia[0, 32:64] @ ib[:, 32:64].T).astype(np.float64) / 4
    assert np.array_equal(out2[0] - out[0], 7 * part)
    assert np.array_equal(out2[1:], out[1:])


def _binades(bs, seed):
    """Two blocks per binade of the block amax, from below the smallest bf16 subnormal to the top of
    the bf16 range (amax mantissa in [1, 1.4) and in [1.6, 2), so CEIL also moves up a binade)."""
    g = np.random.default_rng(seed)
    ks = np.repeat(np.arange(-136, 128), 2)
    mant = np.where(np.arange(len(ks)) % 2 == 0, 1.0, 1.6) + g.uniform(0.0, 0.39, len(ks))
    blocks = g.uniform(-1.0, 1.0, (len(ks), bs)) * np.ldexp(1.0, ks)[:, None]
    blocks[:, 0] = np.ldexp(mant, ks) * g.choice([-1.0, 1.0], len(ks))
    return torch.from_numpy(blocks.reshape(-1, 128).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", ["mxfp4", "mxfp8"])
@pytest.mark.parametrize("rule", ["even", "ceil"])
def test_mx_quantize_every_scale_code_matches_library_construction(orc, fmt, rule):
    # every E8M0 code the rules reach, 0 through 254, including the clamp at -127 for subnormal
    # blocks and the top binade of bf16
    f = orc.MXFP4 if fmt == "mxfp4" else orc.MXFP8
    r = orc.EVEN if rule == "even" else orc.CEIL
    x = _binades(32, 31)
    q, sf = orc.quantize(x, f, r)
    codes_ref, sf_ref = _mx_reference(x, fmt, rule)
    assert np.array_equal(sf, sf_ref)
    assert sf.min() == 0 and sf.max() >= 246
    codes = q if fmt == "mxfp8" else _unpack_fp4(q)
    assert np.array_equal(codes, codes_ref)


@pytest.mark.parametrize("g", [1.0e-30, 3.7e-6, 1.0 / 2688, 1.0, 5.0e20, 2.0 ** 100])
def test_nvfp4_every_binade_matches_fp32_library_construction(orc, g):
    # blocks in every binade against fixed global scales that send scales to 0, saturate them at
    # 448, or leave them in range (subnormal g, where fl(1/d) can overflow, is pinned separately)
    x = _binades(16, 32)
    q, sf = orc.quantize(x, orc.NVFP4, 0, g=g)
    codes_ref, sf_ref = _nvfp4_reference(x, g)
    assert np.array_equal(sf, sf_ref)
    assert np.array_equal(_unpack_fp4(q), codes_ref)


_E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
_E2M1_MIDPOINTS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def _e4m3_positive_table():
    """(exact value, code) for every finite non-negative E4M3 code, decoded by ml_dtypes."""
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x7F is NaN
    vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return [(Fraction(float(v)), int(c)) for v, c in zip(vals, codes)]


def _near(q, points, rel):
    return any(abs(q - p) <= abs(p) * rel for p in points)


@pytest.mark.parametrize("g_kind", ["tensor", "one", "small"])
def test_nvfp4_exact_rounding_away_from_midpoints(orc, g_kind):
    """NVFP4 against its order-free definition, in exact rational arithmetic: the block scale is the
    E4M3 value nearest to amax / (6 g) (saturating at 448), and each element is the E2M1 value
    nearest to x / (dec(s) g), saturating at 6, with x's sign.  Any fp32 order of those steps moves
    the quotients by a few fp32 ulps at most, so wherever an exact quotient lies further than 2^-20
    (relative) from a rounding midpoint the result is fixed whatever the order; the rest are skipped,
    and must be few.  A wrong block size, a global scale applied the other way, a 6 in place of 448
    or a swapped nibble all fail here."""
    x = _adversarial_bf16(16, 512, 77, huge=40.0, bs=16)
    if g_kind == "tensor":
        g, _ = orc.global_scale(x)
    else:
        g = np.float32(1.0 if g_kind == "one" else 3.7e-6)
    q, sf = orc.quantize(x, orc.NVFP4, 0, g=float(g))
    codes = _unpack_fp4(q)
    gq = Fraction(float(g))
    table = _e4m3_positive_table()  # index = code
    e4m3_mid = [(table[i][0] + table[i + 1][0]) / 2 for i in range(len(table) - 1)]
    e2m1_mid = [Fraction(m) for m in _E2M1_MIDPOINTS]
    xf = x.float().numpy().astype(np.float64).reshape(16, -1, 16)
    rel = Fraction(1, 1 << 20)
    n_blocks = xf.shape[0] * xf.shape[1]
    zero_blocks = checked_s = checked_q = skipped_q = 0
    for r in range(xf.shape[0]):
        for b in range(xf.shape[1]):
            blk = xf[r, b]
            amax = Fraction(float(np.abs(blk).max()))
            u = amax / (6 * gq)
            s_code = int(sf[r, b])
            if amax == 0:
                assert s_code == 0
                zero_blocks += 1
            elif u >= 448:
                assert s_code == 0x7E, (r, b)
                checked_s += 1
            elif not _near(u, e4m3_mid, rel):
                best = min(table, key=lambda vc: abs(vc[0] - u))
                assert s_code == best[1], (r, b, float(u))
                checked_s += 1
            dq = table[s_code][0] * gq
            for i in range(16):
                xi = float(blk[i])
                c = int(codes[r, b * 16 + i])
                sign = 8 if math.copysign(1.0, xi) < 0 else 0
                if dq == 0:
                    assert c == sign, (r, b, i)
                    checked_q += 1
                    continue
                v = abs(Fraction(xi)) / dq
                if _near(v, e2m1_mid, rel):
                    skipped_q += 1
                    continue
                mag = 7 if v > 5 else min(range(8), key=lambda k: abs(Fraction(_E2M1_VALUES[k]) - v))
                assert c == (mag | sign), (r, b, i, float(v))
                checked_q += 1
    assert zero_blocks + checked_s >= 0.95 * n_blocks
    assert checked_q >= 0.8 * xf.size and skipped_q <= 0.05 * xf.size
