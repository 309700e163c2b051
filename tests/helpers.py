"""Shared test helpers: tolerance checks and oracle/GPU glue (test infrastructure only)."""
import numpy as np
import torch

import oracle

FMTS = {"mxfp4": oracle.MXFP4, "nvfp4": oracle.NVFP4, "mxfp8": oracle.MXFP8}
RULES = {"even": oracle.EVEN, "ceil": oracle.CEIL}

# fp32 GEMM tolerance: |gpu - ref| <= 2^-20 * sum_k |a_k b_k| (per element).
FP32_REL = 2.0 ** -20


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (8 significant bits); subnormal floor 2^-133."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, np.ldexp(1.0, (e - 7).astype(np.int64)), 2.0 ** -133)


def check_fp32(gpu, ref, abs_sum, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = FP32_REL * abs_sum
    bad = err > bound
    ratio = float(np.max(np.where(bound > 0, err / np.maximum(bound, 1e-300), np.where(err > 0, np.inf, 0.0))))
    assert not bad.any(), "%s: %d of %d outside 2^-20*sum|ab| (worst ratio %.3g)" % (what, bad.sum(), bad.size, ratio)
    return ratio


def check_bf16(gpu, ref, abs_sum, what=""):
    """bf16 output = RNE of an fp32 result that meets the fp32 bound: within 1 bf16 ulp of ref
    plus the fp32 accumulation allowance."""
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = bf16_ulp(ref) + FP32_REL * abs_sum
    bad = err > bound
    assert not bad.any(), "%s: %d of %d outside 1 bf16 ulp (+fp32 allowance); worst err %.3g" % (
        what, bad.sum(), bad.size, float(err[bad].max()) if bad.any() else 0.0)
    # and nearly all are the correctly rounded value or its neighbour
    return float(np.mean(err <= 0.5 * bf16_ulp(ref) + FP32_REL * abs_sum))


def to_np(t):
    return t.detach().cpu().numpy()


def oracle_quantize(x_cpu, fmt, rule, g=1.0):
    return oracle.quantize(x_cpu, FMTS[fmt], RULES[rule], g=float(g))


def gpu_sf_rowmajor(sf_swz, rows, kblocks):
    return oracle.unswizzle(to_np(sf_swz), rows, kblocks)
