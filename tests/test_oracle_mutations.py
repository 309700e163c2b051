"""The oracle's pins against planted mistakes.

Each case copies the oracle (``oracle/oracle.py`` and ``oracle/mxq_oracle.c``) into a temporary
directory, plants one plausible mistake in the C source of the copy (on the CPU: the copy is built
with gcc and loaded through its own ctypes wrapper; the product library is not involved), and
requires at least one of the named pins to fail on it.  A control case runs the same pins on an
unchanged copy, which must pass, so the failures come from the planted mistakes alone.

The mistakes are the kinds the pins are meant to catch: an off-by-one exponent, a strict instead
of a non-strict comparison, a wrong clamp, ties rounded away from zero, a wrong saturation value,
a wrong exponent bias, swapped nibbles, a swizzle that is not a bijection, a dropped global scale,
a dropped term of a sum, a global scale applied the wrong way, a short block, a wrong global
scale constant, swapped activation columns in the weight-only GEMM, bf16 rounding by truncation,
a running maximum that forgets its history, MX elements scaled one binade off, a wrong E8M0 bias
and a dropped sign.  Every planted change keeps all memory accesses
inside their buffers.
"""
import importlib.util
import os
import shutil

import pytest

import test_oracle_fakequant as FQ
import test_oracle_formats as F
import test_oracle_quant as Q
import test_oracle_w4a16 as W

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

# name: (exact text in mxq_oracle.c, replacement, pins that must catch it)
MUTANTS = {
    "even_rule_off_by_one": (
        "        e = floor_log2 - elem_emax;\n",
        "        e = floor_log2 - elem_emax + 1;\n",
        ["mx_exponent_golden", "mx_exponent_exhaustive"]),
    "ceil_rule_non_strict": (
        "        while (amax > ldexp(elem_max, e)) e++;\n",
        "        while (amax >= ldexp(elem_max, e)) e++;\n",
        ["mx_exponent_golden", "mx_exponent_exhaustive"]),
    "exponent_clamp": (
        "    if (e < -127) e = -127;\n",
        "    if (e < -126) e = -126;\n",
        ["mx_exponent_clamp", "mx_exponent_exhaustive"]),
    "ties_away_from_zero": (
        "    double n = rint(a / quantum); /* a / quantum is exact; rint rounds ties to even */\n",
        "    double n = floor(a / quantum + 0.5);\n",
        ["e2m1_tie_table", "e2m1_encode_library"]),
    "e4m3_saturation_value": (
        "uint8_t orc_e4m3_encode(double v) { return (uint8_t)minifloat_encode(v, 4, 3, 7, 448.0); }\n",
        "uint8_t orc_e4m3_encode(double v) { return (uint8_t)minifloat_encode(v, 4, 3, 7, 480.0); }\n",
        ["e4m3_saturates"]),
    "e2m1_bias": (
        "double orc_e2m1_value(uint8_t code) { return minifloat_value(code & 0xFu, 2, 1, 1); }\n",
        "double orc_e2m1_value(uint8_t code) { return minifloat_value(code & 0xFu, 2, 1, 0); }\n",
        ["e2m1_decode"]),
    "nibbles_swapped_on_read": (
        "        uint8_t byte = q[(r * K + k) / 2];\n        elem = orc_e2m1_value(k % 2 == 0 ? (byte & 0xFu) : (byte >> 4));\n    }\n",
        "        uint8_t byte = q[(r * K + k) / 2];\n        elem = orc_e2m1_value(k % 2 == 1 ? (byte & 0xFu) : (byte >> 4));\n    }\n",
        ["fp4_nibble_order", "gemm_mxfp4"]),
    "swizzle_not_a_bijection": (
        "(r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);\n",
        "(r % 32) * 4 + ((r % 128) / 32) * 16 + (c % 4);\n",
        ["swizzle_layout"]),
    "gemm_drops_global_scale": (
        "    double alpha = fmt == ORC_NVFP4 ? gA * gB : 1.0;\n",
        "    double alpha = fmt == ORC_NVFP4 ? gA : 1.0;\n",
        ["gemm_nvfp4"]),
    "gemm_drops_first_term": (
        "            const double* a = g->arow + i * K;\n            for (int64_t k = 0; k < K; k++) {\n",
        "            const double* a = g->arow + i * K;\n            for (int64_t k = 1; k < K; k++) {\n",
        ["gemm_mxfp4", "gemm_exact"]),
    "nvfp4_global_scale_inverted": (
        "        volatile float u = t / g;\n",
        "        volatile float u = t * g;\n",
        ["nvfp4_exact", "nvfp4_library"]),
    "nvfp4_short_block_amax": (
        "    float amax = (float)block_amax(x, 16);\n",
        "    float amax = (float)block_amax(x, 8);\n",
        ["nvfp4_exact", "nvfp4_library"]),
    "global_scale_constant": (
        "    volatile float g = amax / 2688.0f;\n",
        "    volatile float g = amax / 448.0f;\n",
        ["nvfp4_library"]),
    "w4a16_drops_global_scale": (
        "    double alpha = fmt == ORC_NVFP4 ? gB : 1.0;\n",
        "    double alpha = 1.0;\n",
        ["w4a16_nvfp4"]),
    "w4a16_swaps_activation_columns": (
        "        for (int64_t k = 0; k < K; k++) arow[i * K + k] = orc_bf16_value(A[m * K + k]);\n",
        "        for (int64_t k = 0; k < K; k++) arow[i * K + k] = orc_bf16_value(A[m * K + (k ^ 1)]);\n",
        ["w4a16_mxfp4", "w4a16_exact"]),
    "bf16_rounding_truncates": (
        "    uint32_t r = u + 0x7FFFu + ((u >> 16) & 1u);\n",
        "    uint32_t r = u;\n",
        ["f32_to_bf16"]),
    "fake_quant_nibbles_swapped": (
        "                uint8_t byte = q[(r * K + k) / 2];\n                elem = orc_e2m1_value(k % 2 == 0 ",
        "                uint8_t byte = q[(r * K + k) / 2];\n                elem = orc_e2m1_value(k % 2 == 1 ",
        ["fake_quant_mxfp4"]),
    "fake_quant_nvfp4_drops_global_scale": (
        "                volatile float d = (float)orc_e4m3_value(s) * g;\n",
        "                volatile float d = (float)orc_e4m3_value(s);\n",
        ["fake_quant_nvfp4"]),
    "mx_elements_scaled_one_binade_off": (
        "                    double v = ldexp(orc_bf16_value(xb[i]), -e); /* exact */\n",
        "                    double v = ldexp(orc_bf16_value(xb[i]), -e - 1);\n",
        ["mx_quantize_mxfp4", "mx_quantize_mxfp8"]),
    "mx_scale_byte_bias": (
        "                sf[r * kb + b] = (uint8_t)(e + 127);\n",
        "                sf[r * kb + b] = (uint8_t)(e + 128);\n",
        ["mx_quantize_mxfp4", "zero_blocks"]),
    "mx_sign_dropped": (
        "    unsigned sign = signbit(v) ? 1u : 0u;\n",
        "    unsigned sign = 0u;\n",
        ["e2m1_encode_library", "zero_blocks"]),
    "running_max_forgets_history": (
        "    *amax_out = a > amax_in ? a : amax_in;\n",
        "    *amax_out = a;\n",
        ["running_max"]),
}

PINS = {
    "mx_exponent_golden": lambda o: F.test_mx_exponent_golden(o),
    "mx_exponent_exhaustive": lambda o: [F.test_mx_exponent_exhaustive_over_bf16(o, fmt, em, mx, rule)
                                         for fmt, em, mx in (("mxfp4", 2, 6), ("mxfp8", 8, 448))
                                         for rule in ("even", "ceil")],
    "mx_exponent_clamp": lambda o: F.test_mx_exponent_clamp(o),
    "e2m1_tie_table": lambda o: F.test_e2m1_tie_table(o),
    "e2m1_encode_library": lambda o: F.test_e2m1_encode_matches_library_and_bruteforce(o),
    "e2m1_decode": lambda o: F.test_e2m1_decode_all_codes(o),
    "e4m3_saturates": lambda o: F.test_e4m3_encode_saturates(o),
    "fp4_nibble_order": lambda o: Q.test_fp4_nibble_order(o),
    "swizzle_layout": lambda o: Q.test_swizzle_layout(o),
    "gemm_mxfp4": lambda o: Q.test_gemm_matches_numpy_fp64(o, "mxfp4"),
    "gemm_nvfp4": lambda o: Q.test_gemm_matches_numpy_fp64(o, "nvfp4"),
    "gemm_exact": lambda o: Q.test_gemm_exact_integers(o),
    "nvfp4_exact": lambda o: [Q.test_nvfp4_exact_rounding_away_from_midpoints(o, k) for k in ("tensor", "one")],
    "nvfp4_library": lambda o: Q.test_nvfp4_matches_fp32_library_construction(o),
    "w4a16_mxfp4": lambda o: W.test_w4a16_matches_numpy_fp64(o, "mxfp4"),
    "w4a16_nvfp4": lambda o: W.test_w4a16_matches_numpy_fp64(o, "nvfp4"),
    "w4a16_exact": lambda o: W.test_w4a16_exact_integers(o),
    "f32_to_bf16": lambda o: FQ.test_f32_to_bf16_matches_torch(o),
    "fake_quant_mxfp4": lambda o: FQ.test_fake_quantize_equals_dequantized_codes(o, "mxfp4", "even"),
    "fake_quant_nvfp4": lambda o: [FQ.test_nvfp4_fake_quantize_is_fp32_product_then_bf16(o, g)
                                   for g in (1.0 / 2688, 1.0, 3.7e-6)],
    "running_max": lambda o: FQ.test_running_max_oracle(o),
    "mx_quantize_mxfp4": lambda o: [Q.test_mx_quantize_matches_library_construction(o, "mxfp4", r)
                                    for r in ("even", "ceil")],
    "mx_quantize_mxfp8": lambda o: [Q.test_mx_quantize_matches_library_construction(o, "mxfp8", r)
                                    for r in ("even", "ceil")],
    "zero_blocks": lambda o: Q.test_zero_blocks(o),
}


def _oracle_copy(tmp_path, name, old=None, new=None):
    d = tmp_path / name
    d.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "oracle.py"), d / "oracle.py")
    src = open(os.path.join(ORACLE_DIR, "mxq_oracle.c")).read()
    if old is not None:
        assert src.count(old) == 1, "the planted change no longer matches the oracle source: " + name
        src = src.replace(old, new)
    (d / "mxq_oracle.c").write_text(src)
    spec = importlib.util.spec_from_file_location("oracle_copy_" + name, str(d / "oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def test_pins_pass_on_an_unchanged_copy(tmp_path):
    o = _oracle_copy(tmp_path, "control")
    for pin in sorted({p for _, _, pins in MUTANTS.values() for p in pins}):
        PINS[pin](o)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new, pins = MUTANTS[name]
    o = _oracle_copy(tmp_path, name, old, new)
    caught = []
    for pin in pins:
        try:
            PINS[pin](o)
        except AssertionError:
            caught.append(pin)
    assert caught, "no pin caught the planted mistake %r (tried %s)" % (name, ", ".join(pins))
