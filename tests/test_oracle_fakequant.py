"""Pins of the oracle's fake quantization (quantize-dequantize to bf16)."""
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_mx_b200 import synth
from tests.test_oracle_quant import _adversarial_bf16


def test_f32_to_bf16_matches_torch(orc):
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * np.exp(rng.uniform(-80, 80, 20000)),
                        np.array([0.0, -0.0, 1.0, 3.0e38, 1e-40, -1e-44, 1.00390625, 1.01171875])]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f32_to_bf16(float(a)) for a in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt,rule", [("mxfp4", "even"), ("mxfp4", "ceil"), ("mxfp8", "even"), ("mxfp8", "ceil"),
                                      ("nvfp4", "even")])
def test_fake_quantize_equals_dequantized_codes(orc, fmt, rule):
    f = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4, "mxfp8": orc.MXFP8}[fmt]
    r = orc.EVEN if rule == "even" else orc.CEIL
    bs = 16 if fmt == "nvfp4" else 32
    x = _adversarial_bf16(24, 320, 17, huge=3.0e30 if fmt != "nvfp4" else 3.0e6, bs=bs)
    g = 1.0
    if fmt == "nvfp4":
        g, _ = orc.global_scale(x)
    y = orc.fake_quantize(x, f, r, g=float(g))
    q, sf = orc.quantize(x, f, r, g=float(g))
    d = orc.dequantize(q, sf, 320, f, g=float(g))  # fp64 value of each dequantized element
    yv = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double().numpy()
    if fmt == "nvfp4":
        # one fp32 product then one bf16 rounding: within half a bf16 ulp of the exact q*s*g, plus
        # the two fp32 roundings
        assert np.all(np.abs(yv - d) <= np.abs(d) * (2.0 ** -8 + 2.0 ** -22))
    else:
        # MX values have at most 4 significant bits: exactly representable in bf16
        assert np.array_equal(yv, d)
    # idempotent: fake-quantizing the fake-quantized tensor changes no value (value idempotence)
    xy = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16)
    if fmt != "nvfp4":
        y2 = orc.fake_quantize(xy, f, r, g=float(g))
        assert np.array_equal(torch.from_numpy(y2.view(np.int16)).view(torch.bfloat16).double().numpy(), yv)


def test_fake_quantize_zero_and_sign(orc):
    x = torch.zeros(2, 32, dtype=torch.bfloat16)
    x[1] = -0.0
    x[1, 3] = -0.01  # rounds to -0 after scaling by its own block amax? no: it is the block amax
    y = orc.fake_quantize(x, orc.MXFP4, orc.CEIL)
    assert np.all(y[0] == 0)
    yv = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert yv[1, 3] < 0 and np.all(np.signbit(yv[1]))


def test_running_max_oracle(orc):
    x = torch.zeros(2, 32, dtype=torch.bfloat16)
    x[0, 5] = 5.0
    q, sf, new = orc.quantize_running(x, 2688.0)  # g = 1
    qref, sfref = orc.quantize(x, orc.NVFP4, 0, g=1.0)
    assert new == np.float32(5.0) or new == np.float32(2688.0)
    assert new == np.float32(2688.0)  # running max keeps the larger state
    assert np.array_equal(q, qref) and np.array_equal(sf, sfref)
    q2, sf2, new2 = orc.quantize_running(x, 1.0)
    assert new2 == np.float32(5.0)
    g = np.float32(1.0) / np.float32(2688.0)
    q3, sf3 = orc.quantize(x, orc.NVFP4, 0, g=float(g))
    assert np.array_equal(q2, q3) and np.array_equal(sf2, sf3)


def _binades(bs, seed):
    """Two blocks per binade of the block amax, from below the smallest bf16 subnormal to the top of
    the bf16 range (amax mantissa in [1, 1.4) and in [1.6, 2), so CEIL also moves up a binade)."""
    g = np.random.default_rng(seed)
    ks = np.repeat(np.arange(-136, 128), 2)
    mant = np.where(np.arange(len(ks)) % 2 == 0, 1.0, 1.6) + g.uniform(0.0, 0.39, len(ks))
    blocks = g.uniform(-1.0, 1.0, (len(ks), bs)) * np.ldexp(1.0, ks)[:, None]
    blocks[:, 0] = np.ldexp(mant, ks) * g.choice([-1.0, 1.0], len(ks))
    return torch.from_numpy(blocks.reshape(-1, 128).astype(np.float32)).to(torch.bfloat16)


def _bits16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("fmt,rule", [("mxfp4", "even"), ("mxfp4", "ceil"), ("mxfp8", "even"), ("mxfp8", "ceil")])
def test_mx_fake_quantize_every_scale_code_is_the_bf16_cast(orc, fmt, rule):
    # every E8M0 code the formats reach (0 through 254): an MX value elem * 2^e has at most 4
    # significant bits, so its bf16 encoding is torch's bf16 cast of the exact fp64 value (inf where
    # it exceeds the bf16 range, as a single fp32 product rounds it)
    f = orc.MXFP4 if fmt == "mxfp4" else orc.MXFP8
    r = orc.EVEN if rule == "even" else orc.CEIL
    x = _binades(32, 21)
    q, sf = orc.quantize(x, f, r)
    assert sf.min() == 0 and sf.max() >= 246
    d = orc.dequantize(q, sf, 128, f)
    expect = _bits16(torch.from_numpy(d).to(torch.bfloat16))
    assert np.array_equal(orc.fake_quantize(x, f, r), expect)


@pytest.mark.parametrize("g", [2.0 ** -140, 1.0e-30, 3.7e-6, 1.0 / 2688, 1.0, 5.0e20, 2.0 ** 100])
def test_nvfp4_fake_quantize_is_fp32_product_then_bf16(orc, g):
    # the NVFP4 decode fl32(elem * fl32(dec(s) * g)), then bf16 RNE, rebuilt from library decoders
    # (ml_dtypes E2M1 and E4M3) and numpy fp32 arithmetic, over blocks in every binade and global
    # scales that make d subnormal, overflow 1/d, or are plain
    import ml_dtypes
    x = _binades(16, 22)
    g32 = np.float32(g)
    q, sf = orc.quantize(x, orc.NVFP4, orc.EVEN, g=float(g32))
    codes = np.stack([q & 0xF, q >> 4], -1).reshape(q.shape[0], -1)
    elem = codes.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    dec = sf.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    d = (dec * g32).astype(np.float32)
    prod = (elem * np.repeat(d, 16, axis=1)).astype(np.float32)
    expect = _bits16(torch.from_numpy(prod).to(torch.bfloat16))
    assert np.array_equal(orc.fake_quantize(x, orc.NVFP4, orc.EVEN, g=float(g32)), expect)
