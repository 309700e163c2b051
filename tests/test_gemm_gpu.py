"""GPU parity of the tcgen05 block-scaled GEMM (mxq_gemm) and the fused linear (mxq_linear)
against the oracle's fp64 GEMM of the dequantized operands.

Tolerance: fp32 output |gpu - ref| <= 2^-20 * sum_k |a_k b_k|; bf16 output within one bf16 ulp of
ref on top of that fp32 allowance."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth
from tests.helpers import FMTS, RULES, check_bf16, check_fp32, oracle_quantize, to_np

pytestmark = pytest.mark.gpu


def _quant_pair(A, W, fmt, a_rule, w_rule):
    gA = gW = 1.0
    if fmt == "nvfp4":
        gA, _ = oracle.global_scale(A)
        gW, _ = oracle.global_scale(W)
    Aq, Asf = oracle_quantize(A, fmt, a_rule, gA)
    Wq, Wsf = oracle_quantize(W, fmt, w_rule, gW)
    return (Aq, Asf, float(gA)), (Wq, Wsf, float(gW))


def _gpu_gemm(a, w, M, N, K, fmt, out_dtype):
    (Aq, Asf, gA), (Wq, Wsf, gW) = a, w
    dev = lambda z: torch.from_numpy(np.ascontiguousarray(z)).cuda()
    g_a = torch.tensor([gA], dtype=torch.float32, device="cuda")
    g_w = torch.tensor([gW], dtype=torch.float32, device="cuda")
    out = mxq.gemm(dev(Aq), dev(oracle.swizzle(Asf)), dev(Wq), dev(oracle.swizzle(Wsf)), M, N, K, fmt,
                   out_dtype=out_dtype, g_A=g_a, g_B=g_w)
    torch.cuda.synchronize()
    return out.double().cpu().numpy() if out_dtype == torch.bfloat16 else to_np(out).astype(np.float64)


# M <= 128 with several K stages runs the split-K cluster kernel; M > 128 the CTA-pair kernel; M <= 128
# with more 128-row weight tiles than SMs the 128 x 256 one-CTA kernel (the last two shapes)
SHAPES = [(1, 1, 64), (16, 256, 256), (128, 128, 128), (200, 300, 320), (129, 520, 1024), (300, 257, 576),
          (64, 96, 5120), (512, 768, 192), (100, 1000, 2048), (128, 4096, 512), (1024, 96, 1024),
          (40, 19200, 256), (7, 19000, 512)]


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES)
def test_gemm_matches_oracle(fmt, out_dtype, shape):
    M, N, K = shape
    if fmt == "mxfp8" and K % 32:
        pytest.skip()
    A = synth.random_bf16((M, K), M + 3 * N + K, std=1.0)
    W = synth.random_bf16((N, K), M + 5 * N + K, std=0.02)
    a, w = _quant_pair(A, W, fmt, "ceil", "even")
    ref, abs_sum = oracle.gemm(a[0], a[1], w[0], w[1], M, N, K, FMTS[fmt], gA=a[2], gB=w[2])
    gpu = _gpu_gemm(a, w, M, N, K, fmt, out_dtype)
    if out_dtype == torch.float32:
        check_fp32(gpu, ref, abs_sum, "%s %s" % (fmt, shape))
    else:
        check_bf16(gpu, ref, abs_sum, "%s %s" % (fmt, shape))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
def test_gemm_unit_scales_exact(fmt):
    """Unit scales and small integer-valued codes: every partial sum is exact in fp32, so the
    GPU result must equal the oracle exactly (pins operand layout and nibble order)."""
    M, N, K = 130, 260, 512
    rng = np.random.default_rng(7)
    bs = 16 if fmt == "nvfp4" else 32
    if fmt == "mxfp8":
        Aq = rng.integers(0, 256, (M, K), dtype=np.uint8)
        Wq = rng.integers(0, 256, (N, K), dtype=np.uint8)
        # normal E4M3 codes with exponent field 8 only: |v| in [2, 3.75], multiples of 1/4
        Aq = (Aq & 0x87) | 0x40
        Wq = (Wq & 0x87) | 0x40
        one = 127
    else:
        Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
        Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
        one = 127 if fmt == "mxfp4" else 0x38  # E8M0 1.0 or E4M3 1.0
    Asf = np.full((M, K // bs), one, np.uint8)
    Wsf = np.full((N, K // bs), one, np.uint8)
    ref, abs_sum = oracle.gemm(Aq, Asf, Wq, Wsf, M, N, K, FMTS[fmt])
    gpu = _gpu_gemm((Aq, Asf, 1.0), (Wq, Wsf, 1.0), M, N, K, fmt, torch.float32)
    assert np.array_equal(gpu, ref), "max abs diff %g" % np.abs(gpu - ref).max()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
def test_gemm_scale_placement(fmt):
    """Distinct power-of-two scales per (row, block) on one operand at a time: pins how the
    swizzled scale tiles map to rows and K blocks inside the MMA."""
    M, N, K = 256, 256, 1024
    bs = 16 if fmt == "nvfp4" else 32
    rng = np.random.default_rng(3)
    A = synth.random_bf16((M, K), 21)
    W = synth.random_bf16((N, K), 22, std=0.02)
    a, w = _quant_pair(A, W, fmt, "even", "even")
    for side in ("A", "B"):
        Aq, Asf, gA = a
        Wq, Wsf, gW = w
        if fmt == "nvfp4":
            codes = np.array([0x30, 0x38, 0x40, 0x48, 0x28], np.uint8)  # 0.5, 1, 2, 4, 0.25
        else:
            codes = np.array([125, 126, 127, 128, 129, 130], np.uint8)
        if side == "A":
            Asf = rng.choice(codes, Asf.shape).astype(np.uint8)
        else:
            Wsf = rng.choice(codes, Wsf.shape).astype(np.uint8)
        ref, abs_sum = oracle.gemm(Aq, Asf, Wq, Wsf, M, N, K, FMTS[fmt], gA=gA, gB=gW)
        gpu = _gpu_gemm((Aq, Asf, gA), (Wq, Wsf, gW), M, N, K, fmt, torch.float32)
        check_fp32(gpu, ref, abs_sum, "%s scales on %s" % (fmt, side))


@pytest.mark.parametrize("fmt,M,N,K", [("mxfp4", 16, 256, 256), ("mxfp4", 200, 333, 640), ("nvfp4", 130, 520, 1024),
                                       ("mxfp8", 64, 96, 512), ("mxfp4", 32, 256, 1280), ("nvfp4", 64, 384, 1024),
                                       ("mxfp8", 100, 200, 640)])
def test_linear_matches_oracle(fmt, M, N, K):
    """mxq_linear (dynamic activation quantization + GEMM) == oracle quantize + fp64 GEMM."""
    A = synth.random_bf16((M, K), 99 + M, std=1.0)
    W = synth.random_bf16((N, K), 98 + N, std=0.02)
    a, w = _quant_pair(A, W, fmt, "ceil", "even")
    ref, abs_sum = oracle.gemm(a[0], a[1], w[0], w[1], M, N, K, FMTS[fmt], gA=a[2], gB=w[2])
    Wd = W.cuda()
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(Wd)
        g_a, _ = mxq.global_scale(A.cuda())
    Wq, Wsf = mxq.quantize(Wd, fmt, "even", global_scale=g_w, layout=mxq.SF_SWIZZLED)
    for out_dtype in (torch.float32, torch.bfloat16):
        out = mxq.linear(A.cuda(), Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=out_dtype, g_W=g_w, g_A=g_a)
        torch.cuda.synchronize()
        gpu = out.double().cpu().numpy()
        if out_dtype == torch.float32:
            check_fp32(gpu, ref, abs_sum, "linear %s" % fmt)
        else:
            check_bf16(gpu, ref, abs_sum, "linear %s" % fmt)


@pytest.mark.parametrize("fmt,rule", [("mxfp4", "ceil"), ("mxfp4", "even"), ("nvfp4", "ceil"), ("mxfp8", "ceil"),
                                      ("mxfp8", "even")])
@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (32, 512, 2048), (17, 300, 320), (7, 96, 5120), (100, 300, 320),
                                   (128, 640, 768), (9, 33000, 320), (1, 20001, 256)])
def test_linear_one_launch_equals_quantize_then_gemm(fmt, rule, M, N, K):
    """Up to 32 tokens: mxq_linear's GEMM quantizes the activations itself (one launch).  Its output
    equals quantizing with mxq_quantize and multiplying with mxq_gemm, bit for bit, including a K
    tail that leaves the last stage partly empty (K = 320), ragged and single-token problems; the
    M = 100 and 128 cases take the two-launch path.  N = 33000 and 20001 have more weight tiles
    than K splits can use: 256 weight rows per CTA, no K split, a last tile that is partly (N =
    33000) or half (N = 20001, also not a multiple of 8: direct stores) past N."""
    if fmt == "mxfp8" and K % 32:
        pytest.skip("K")
    A = synth.random_bf16((M, K), 7 + M + K, std=1.0).cuda()
    W = synth.random_bf16((N, K), 8 + N, std=0.02).cuda()
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        g_a, _ = mxq.global_scale(A)
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    Aq, Asf = mxq.quantize(A, fmt, rule, global_scale=g_a)
    for out_dtype in (torch.float32, torch.bfloat16):
        two = mxq.gemm(Aq, Asf, Wq, Wsf, M, N, K, fmt, out_dtype=out_dtype, g_A=g_a, g_B=g_w)
        one = mxq.linear(A, Wq, Wsf, N, fmt, act_rule=rule, out_dtype=out_dtype, g_W=g_w, g_A=g_a)
        torch.cuda.synchronize()
        assert torch.equal(one.view(torch.int32 if out_dtype == torch.float32 else torch.int16),
                           two.view(torch.int32 if out_dtype == torch.float32 else torch.int16)), (fmt, rule, M, N, K)
    assert mxq.mxq_device_status(reset=True) == 0


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("M,N,K", [(32, 512, 2048), (5, 33000, 320)])
def test_linear_one_launch_x_16_byte_aligned(fmt, M, N, K):
    """The API promises 16-byte alignment of x, which is all the few-token kernel's 16-byte token
    loads need.  x here starts 16 bytes into an allocation (not 32-byte aligned); the output equals
    mxq_quantize + mxq_gemm bit for bit, and the same call on an aligned copy of x."""
    base = synth.random_bf16((M * K + 8,), 11 + M + K, std=1.0).cuda()
    A = base[8:].view(M, K)
    assert A.data_ptr() % 32 == 16
    W = synth.random_bf16((N, K), 12 + N, std=0.02).cuda()
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        g_a, _ = mxq.global_scale(A)
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    Aq, Asf = mxq.quantize(A, fmt, "ceil", global_scale=g_a)
    two = mxq.gemm(Aq, Asf, Wq, Wsf, M, N, K, fmt, out_dtype=torch.float32, g_A=g_a, g_B=g_w)
    one = mxq.linear(A, Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=torch.float32, g_W=g_w, g_A=g_a)
    aligned = mxq.linear(A.clone(), Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=torch.float32, g_W=g_w, g_A=g_a)
    torch.cuda.synchronize()
    assert mxq.linear_kernel_count(M, N, K, fmt) == 1
    assert torch.equal(one.view(torch.int32), two.view(torch.int32))
    assert torch.equal(one.view(torch.int32), aligned.view(torch.int32))
    assert mxq.mxq_device_status(reset=True) == 0


@pytest.mark.parametrize("fmt,rule", [("mxfp4", "ceil"), ("mxfp4", "even"), ("nvfp4", "even"), ("mxfp8", "even"),
                                      ("mxfp8", "ceil")])
@pytest.mark.parametrize("M,N,K", [(33, 96, 512), (129, 1, 640), (300, 128, 320), (1000, 100, 1024), (257, 17, 5120),
                                   (4000, 96, 256), (45, 64, 768)])
def test_linear_small_n_matches_oracle(fmt, rule, M, N, K):
    """More than 32 tokens and N <= 128: mxq_linear is one launch, the small-N kernel quantizing each
    128-row activation tile on its way into the tensor cores (K split over a cluster).  Checked
    against the oracle from the bf16 inputs, fp32 and bf16 out, with ragged M tiles, N = 1 and
    N < 128 column tails, a K tail that leaves the last stage partly empty (K = 320) and one K
    stage only (K = 256 for FP4: no split).  Clusters of 2 and 3 CTAs share the reduction by
    32-row sub-partition; (45, 64, 768) splits K three ways over a tile whose last two
    sub-partitions hold no valid row, so one CTA receives and stores nothing."""
    if fmt == "mxfp8" and K % 32:
        pytest.skip("K")
    assert mxq.linear_kernel_count(M, N, K, fmt) == 1
    A = synth.random_bf16((M, K), 31 + M + K, std=1.0)
    W = synth.random_bf16((N, K), 37 + N, std=0.02)
    a, w = _quant_pair(A, W, fmt, rule, "even")
    ref, abs_sum = oracle.gemm(a[0], a[1], w[0], w[1], M, N, K, FMTS[fmt], gA=a[2], gB=w[2])
    Wd, Ad = W.cuda(), A.cuda()
    g_w = g_a = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(Wd)
        g_a, _ = mxq.global_scale(Ad)
    Wq, Wsf = mxq.quantize(Wd, fmt, "even", global_scale=g_w)
    for out_dtype in (torch.float32, torch.bfloat16):
        out = mxq.linear(Ad, Wq, Wsf, N, fmt, act_rule=rule, out_dtype=out_dtype, g_W=g_w, g_A=g_a)
        torch.cuda.synchronize()
        gpu = out.double().cpu().numpy()
        if out_dtype == torch.float32:
            check_fp32(gpu, ref, abs_sum, "small-N linear %s %s" % (fmt, (M, N, K)))
        else:
            check_bf16(gpu, ref, abs_sum, "small-N linear %s %s" % (fmt, (M, N, K)))
    assert mxq.mxq_device_status(reset=True) == 0


def test_linear_kernel_count():
    """mxq_linear_kernel_count reports the one-launch path exactly where the bit-equality test above
    exercises it: up to 32 tokens with several K splits."""
    assert mxq.linear_kernel_count(32, 5120, 5120, "mxfp4") == 1
    assert mxq.linear_kernel_count(1, 256, 1024, "nvfp4") == 1
    assert mxq.linear_kernel_count(7, 96, 5120, "mxfp8") == 1
    assert mxq.linear_kernel_count(100, 300, 320, "mxfp4") == 2
    assert mxq.linear_kernel_count(8192, 34816, 5120, "mxfp4") == 2
    assert mxq.linear_kernel_count(32, 34816, 5120, "mxfp4") == 1  # 256 weight rows per CTA, one wave
    assert mxq.linear_kernel_count(32, 151936, 5120, "mxfp4") == 2  # more than one wave: quantizer + GEMM
    assert mxq.linear_kernel_count(8192, 96, 5120, "mxfp8") == 1  # small N: the GEMM quantizes its rows
    assert mxq.linear_kernel_count(8192, 129, 5120, "mxfp8") == 2


def test_tiny_config_full():
    """The tiny MXFP4 W4A4 linear problem: every output element, fp32 out."""
    cfg = synth.CONFIGS["tiny"]
    A, W = synth.make_inputs("tiny")
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    a, w = _quant_pair(A, W, "mxfp4", "ceil", "even")
    ref, abs_sum = oracle.gemm(a[0], a[1], w[0], w[1], M, N, K, oracle.MXFP4)
    Wq, Wsf = mxq.quantize(W.cuda(), "mxfp4", "even")
    out = mxq.linear(A.cuda(), Wq, Wsf, N, "mxfp4", act_rule="ceil", out_dtype=torch.float32)
    torch.cuda.synchronize()
    check_fp32(to_np(out).astype(np.float64), ref, abs_sum, "tiny")


def test_bounded_wait_selftest():
    """A kernel waiting on a barrier nothing completes gives up after its limit and reports
    MXQ_ERR_TIMEOUT through the status word; the context stays usable."""
    mxq.mxq_device_status(reset=True)
    mxq.mxq_selftest_timeout(20_000_000)  # 20 ms
    st = mxq.mxq_device_status(reset=True)
    assert st == 0x100 + 99
    assert mxq.mxq_device_status(reset=False) == 0
    x = torch.ones(4, 64, dtype=torch.bfloat16, device="cuda")
    q, sf = mxq.quantize(x, "mxfp4", "ceil", layout=mxq.SF_ROWMAJOR)
    torch.cuda.synchronize()
    assert int(sf[0, 0]) == 125  # amax 1 -> CEIL e = -2


# fixed seeds of the sampled rows and columns, one per problem (reproducible across processes)
SAMPLE_SEED = {"decode": 2001, "prefill_gate_up": 2002, "down_nvfp4": 2003, "attn_mxfp8": 2004, "lm_head": 2005,
               "in_proj_ba": 2006}


def _sample(total, tile, n, gen):
    """About n seeded indices in [0, total): the same number in every `tile`-wide stretch (at least
    one), so every output tile the kernels emit is visited, plus the last index (the tail)."""
    if total <= n:
        return np.arange(total, dtype=np.int64)
    tiles = (total + tile - 1) // tile
    per = max(1, -(-n // tiles))
    idx = set()
    for t in range(tiles):
        lo, hi = t * tile, min(total, (t + 1) * tile)
        idx.update(torch.randint(lo, hi, (min(per, hi - lo),), generator=gen).tolist())
    idx.add(total - 1)
    return np.array(sorted(idx), dtype=np.int64)


@pytest.mark.parametrize("name", ["decode", "prefill_gate_up", "down_nvfp4", "attn_mxfp8", "lm_head", "in_proj_ba"])
def test_linear_full_size(name):
    """Each full-size problem through mxq_linear in the bench's launch configuration (weights
    quantized on the GPU, activations quantized inside the call), checked against the oracle run on
    the bf16 inputs alone:
      - every quantized byte of A and W (mxq_quantize, the quantizer mxq_linear runs) equals the
        oracle's;
      - outputs: about 128 seeded rows (the same number in every 256-row M tile, plus the last row)
        times ALL N columns, and ALL M rows times about 128 seeded columns (the same number in every
        256-column N tile, plus the last column); every output when M or N is small (decode: all of
        it).  Together they visit every output tile, the last partial waves and the N tail."""
    cfg = synth.CONFIGS[name]
    M, N, K, fmt = cfg["M"], cfg["N"], cfg["K"], cfg["fmt"]
    A, W = synth.make_inputs(name, device="cuda")
    g_w = g_a = None
    gA = gW = 1.0
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
        g_a, _ = mxq.global_scale(A)
        gW_ref, _ = oracle.global_scale(W.cpu())
        gA_ref, _ = oracle.global_scale(A.cpu())
        assert to_np(g_w)[0] == gW_ref and to_np(g_a)[0] == gA_ref
        gA, gW = float(gA_ref), float(gW_ref)
    Wq, Wsf = mxq.quantize(W, fmt, cfg["w_rule"], global_scale=g_w, layout=mxq.SF_SWIZZLED)
    out_dtype = torch.float32 if cfg["out"] == "fp32" else torch.bfloat16
    out = mxq.linear(A, Wq, Wsf, N, fmt, act_rule=cfg["a_rule"], out_dtype=out_dtype, g_W=g_w, g_A=g_a)
    Aq_gpu, Asf_gpu = mxq.quantize(A, fmt, cfg["a_rule"], global_scale=g_a, layout=mxq.SF_SWIZZLED)
    torch.cuda.synchronize()
    assert mxq.mxq_device_status(reset=True) == 0
    bs = 16 if fmt == "nvfp4" else 32

    # every quantized byte of both operands (oracle threads over row ranges; the bytes do not depend on it)
    Wq_ref, Wsf_ref = oracle.quantize(W.cpu(), FMTS[fmt], RULES[cfg["w_rule"]], g=gW, threads=None)
    assert np.array_equal(to_np(Wq), Wq_ref), "%s: weight codes differ" % name
    assert np.array_equal(to_np(Wsf), oracle.swizzle(Wsf_ref)), "%s: weight scales differ" % name
    Aq_ref, Asf_ref = oracle.quantize(A.cpu(), FMTS[fmt], RULES[cfg["a_rule"]], g=gA, threads=None)
    assert np.array_equal(to_np(Aq_gpu), Aq_ref), "%s: activation codes differ" % name
    assert np.array_equal(to_np(Asf_gpu), oracle.swizzle(Asf_ref)), "%s: activation scales differ" % name
    del Wq, Wsf, Aq_gpu, Asf_gpu, W, A

    check = check_fp32 if out_dtype == torch.float32 else check_bf16
    gen = torch.Generator().manual_seed(SAMPLE_SEED[name])
    rows = _sample(M, 256, 128, gen)
    cols = _sample(N, 256, 128, gen)
    # seeded rows x all columns
    ref, abs_sum = oracle.gemm(Aq_ref, Asf_ref, Wq_ref, Wsf_ref, M, N, K, FMTS[fmt], gA=gA, gB=gW, rows=rows,
                               threads=None)
    check(out[torch.from_numpy(rows).cuda()].double().cpu().numpy(), ref, abs_sum, "%s rows x all N" % name)
    if len(rows) < M:
        # all rows x seeded columns, as the transposed product (the fp64 sums are the same terms)
        ref_t, abs_t = oracle.gemm(Wq_ref, Wsf_ref, Aq_ref, Asf_ref, N, M, K, FMTS[fmt], gA=gW, gB=gA, rows=cols,
                                   threads=None)
        check(out[:, torch.from_numpy(cols).cuda()].double().cpu().numpy(), ref_t.T, abs_t.T,
              "%s all M x columns" % name)
