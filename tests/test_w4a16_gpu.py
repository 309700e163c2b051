"""GPU parity of the weight-only (W4A16) GEMM mxq_gemm_w4a16 against the oracle's fp64
weight-only GEMM (bf16 activations times dequantized MXFP4 / NVFP4 weights).

Tolerance: as for the W4A4 GEMM, fp32 output |gpu - ref| <= 2^-20 * sum_k |a_k w_k|; bf16 output
within one bf16 ulp of ref on top of that allowance.  The dequantized weights are exact in bf16, so
the only rounding is the fp32 accumulation (and the bf16 store)."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth
from tests.helpers import FMTS, RULES, check_bf16, check_fp32, oracle_quantize, to_np

pytestmark = pytest.mark.gpu


def _weights(W, fmt):
    gW = 1.0
    if fmt == "nvfp4":
        gW, _ = oracle.global_scale(W)
    Wq, Wsf = oracle_quantize(W, fmt, "even", gW)
    return Wq, Wsf, float(gW)


def _gpu_w4a16(A, w, N, fmt, out_dtype):
    Wq, Wsf, gW = w
    dev = lambda z: torch.from_numpy(np.ascontiguousarray(z)).cuda()
    g_w = torch.tensor([gW], dtype=torch.float32, device="cuda")
    out = mxq.gemm_w4a16(A.cuda(), dev(Wq), dev(oracle.swizzle(Wsf)), N, fmt, g_W=g_w, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return out.double().cpu().numpy() if out_dtype == torch.bfloat16 else to_np(out).astype(np.float64)


# M <= 128 runs 128 x 64 tiles with one accumulator; M > 128 256 x 256 tiles with two
SHAPES = [(1, 1, 64), (16, 256, 256), (128, 128, 128), (200, 300, 320), (129, 520, 1024), (300, 257, 576),
          (64, 96, 5120), (512, 768, 192), (100, 1000, 2048), (1024, 96, 1024), (777, 1111, 704),
          (32, 19200, 256), (100, 9600, 512),  # these two: more weight tiles than SMs
          (17, 1024, 4096), (5, 300, 1600),  # K split over 4 and 3 CTAs at 32 tokens, a ragged last K stage
          (32, 1024, 2304), (48, 512, 2304)]  # 9 K stages: 3 splits of 3 (4 splits would leave one empty)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES)
def test_w4a16_matches_oracle(fmt, out_dtype, shape):
    M, N, K = shape
    A = synth.random_bf16((M, K), 3 * M + N + K, std=1.0)
    W = synth.random_bf16((N, K), M + 7 * N + K, std=0.02)
    w = _weights(W, fmt)
    ref, abs_sum = oracle.gemm_w4a16(A, w[0], w[1], M, N, K, FMTS[fmt], gB=w[2])
    gpu = _gpu_w4a16(A, w, N, fmt, out_dtype)
    if out_dtype == torch.float32:
        check_fp32(gpu, ref, abs_sum, "%s %s" % (fmt, shape))
    else:
        check_bf16(gpu, ref, abs_sum, "%s %s" % (fmt, shape))


@pytest.mark.parametrize("M", [40, 300])
def test_w4a16_exact_integers(M):
    """Unit scales, small integer activations: every partial sum is exact in fp32, so the GPU
    equals the oracle exactly (pins the nibble order, the B layout and the dequantization)."""
    N, K = 200, 384
    rng = np.random.default_rng(M)
    a_int = rng.integers(-8, 9, (M, K)).astype(np.float32)
    A = torch.from_numpy(a_int).to(torch.bfloat16)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Wsf = np.full((N, K // 32), 127, np.uint8)
    ref, _ = oracle.gemm_w4a16(A, Wq, Wsf, M, N, K, oracle.MXFP4)
    gpu = _gpu_w4a16(A, (Wq, Wsf, 1.0), N, "mxfp4", torch.float32)
    assert np.array_equal(gpu, ref), "max abs diff %g" % np.abs(gpu - ref).max()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("M", [64, 256])
def test_w4a16_scale_placement(fmt, M):
    """Distinct power-of-two block scales per (row, block) of W: pins how the swizzled scale tiles
    map to weight rows and K blocks, including 64-row tiles that start inside a scale tile."""
    N, K = 320, 512
    bs = 16 if fmt == "nvfp4" else 32
    rng = np.random.default_rng(13)
    A = synth.random_bf16((M, K), 51)
    W = synth.random_bf16((N, K), 52, std=0.02)
    Wq, Wsf, gW = _weights(W, fmt)
    codes = np.array([0x30, 0x38, 0x40, 0x48, 0x28], np.uint8) if fmt == "nvfp4" else \
        np.array([125, 126, 127, 128, 129, 130], np.uint8)
    Wsf = rng.choice(codes, (N, K // bs)).astype(np.uint8)
    ref, abs_sum = oracle.gemm_w4a16(A, Wq, Wsf, M, N, K, FMTS[fmt], gB=gW)
    gpu = _gpu_w4a16(A, (Wq, Wsf, gW), N, fmt, torch.float32)
    check_fp32(gpu, ref, abs_sum, "%s scales" % fmt)


@pytest.mark.parametrize("M", [130, 32, 100])
@pytest.mark.parametrize("codes,a_scale", [((0, 1, 2, 3, 4), 2.0 ** 100), ((248, 249, 250, 251, 252), 2.0 ** -100),
                                           ((126, 127, 128, 129, 130), 1.0), ((2, 3, 127, 128), 1.0)])
def test_w4a16_extreme_mx_scales(M, codes, a_scale):
    """E8M0 scales across the range: codes 2 ... 128 (2^-125 ... 2) dequantize through the integer
    multiply path, the others through the exact fp32 path, chosen per warp; every M covers another
    kernel (one dequantizing into shared memory, two into tensor memory).  Activations are scaled
    so that the products and sums stay normal fp32 numbers."""
    N, K = 96, 256
    rng = np.random.default_rng(codes[0] + M)
    A = (synth.random_bf16((M, K), 61).float() * a_scale).to(torch.bfloat16)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Wsf = rng.choice(np.array(codes, np.uint8), (N, K // 32)).astype(np.uint8)
    ref, abs_sum = oracle.gemm_w4a16(A, Wq, Wsf, M, N, K, oracle.MXFP4)
    gpu = _gpu_w4a16(A, (Wq, Wsf, 1.0), N, "mxfp4", torch.float32)
    check_fp32(gpu, ref, abs_sum, "extreme scales %s" % (codes,))


def test_w4a16_rejects_mxfp8_and_bad_shapes():
    A = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(8, 32, dtype=torch.uint8, device="cuda")
    Wsf = torch.zeros(mxq.sf_bytes(8, 64, "mxfp4"), dtype=torch.uint8, device="cuda")
    with pytest.raises(mxq.MxqError):
        mxq.gemm_w4a16(A, Wq, Wsf, 8, "mxfp8")
    with pytest.raises(mxq.MxqError):
        mxq.gemm_w4a16(torch.zeros(4, 96, dtype=torch.bfloat16, device="cuda"), Wq, Wsf, 8, "mxfp4")


@pytest.mark.parametrize("name,M", [("decode", 32), ("prefill_gate_up", 8192)])
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_w4a16_full_size_sampled(name, M, fmt):
    """Full-size weight-only problems (the decode and prefill gate+up shapes, weights quantized on
    the GPU); a seeded sample of outputs is recomputed by the oracle from the bf16 inputs alone."""
    cfg = synth.CONFIGS[name]
    N, K = cfg["N"], cfg["K"]
    A, W = synth.make_inputs(name, device="cuda")
    g_w = None
    gW = 1.0
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        gW, _ = oracle.global_scale(W.cpu())
        assert to_np(g_w)[0] == gW
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w, layout=mxq.SF_SWIZZLED)
    out = mxq.gemm_w4a16(A, Wq, Wsf, N, fmt, g_W=g_w)
    torch.cuda.synchronize()
    gen = torch.Generator().manual_seed(M + N)
    rows = sorted(set(torch.randint(0, M, (min(M, 48),), generator=gen).tolist()) | {M - 1})
    cols = sorted(set(torch.randint(0, N, (48,), generator=gen).tolist()) | {N - 1})
    Wq_ref, Wsf_ref = oracle_quantize(W[cols].cpu(), fmt, "even", gW)
    ref, abs_sum = oracle.gemm_w4a16(A[rows].cpu(), Wq_ref, Wsf_ref, len(rows), len(cols), K, FMTS[fmt], gB=float(gW))
    gpu = out[rows][:, cols].double().cpu().numpy()
    check_bf16(gpu, ref, abs_sum, "%s %s" % (name, fmt))
