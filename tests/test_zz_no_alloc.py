"""The allocation-free linear entry point (mxq_linear_noalloc).

Callers that may not allocate device memory (plugins that only receive their input and output
buffers, processes under a fixed device-memory cap) use mxq_linear_noalloc, which takes the
activation workspace from a static array inside the library instead of from the caller.  These
tests call it through the C ABI and check its output against the regular mxq_linear on the same
inputs for two calls in a row (the second with fewer tokens and different data, so stale scratch
contents would show).  Both calls run the same kernels on the same bytes, so the outputs must be
bit-identical; the oracle's GEMM tolerance is checked as well.  This file is collected last on
purpose: a failure here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth
from tests.helpers import FMTS, check_bf16, check_fp32, oracle_quantize

pytestmark = pytest.mark.gpu


def _noalloc(x, Wq, Wsf, N, fmt, rule, out, g_w=None, g_a=None):
    M, K = x.shape
    ot = mxq.OUT_FP32 if out.dtype == torch.float32 else mxq.OUT_BF16
    p = lambda t: None if t is None else t.data_ptr()
    return mxq.lib().mxq_linear_noalloc(p(x), p(Wq), p(Wsf), p(g_w), p(g_a), M, N, K, mxq.FMT[fmt],
                                        mxq.RULE[rule], ot, p(out), torch.cuda.current_stream().cuda_stream)


# N = 384 with 200 and 37 tokens takes the quantizer + GEMM path (the array holds the quantized
# activations); N = 96 and 17 tokens take the one-launch kernels that quantize inside the GEMM
@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,calls", [(384, ((200, 11), (37, 12))), (96, ((200, 13), (17, 14)))])
def test_noalloc_matches_linear_two_calls(fmt, out_dtype, N, calls):
    K = 1024
    W = synth.random_bf16((N, K), 5, std=0.02).cuda()
    g_w = None
    if fmt == "nvfp4":
        g_w, _ = mxq.global_scale(W)
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w, layout=mxq.SF_SWIZZLED)
    Wq_ref, Wsf_ref = oracle_quantize(W.cpu(), fmt, "even", float(g_w.item()) if g_w is not None else 1.0)
    for M, seed in calls:
        A = synth.random_bf16((M, K), seed).cuda()
        g_a = None
        if fmt == "nvfp4":
            g_a, _ = mxq.global_scale(A)
        expect = mxq.linear(A, Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=out_dtype, g_W=g_w, g_A=g_a)
        out = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        assert _noalloc(A, Wq, Wsf, N, fmt, "ceil", out, g_w, g_a) == 0
        torch.cuda.synchronize()
        # the oracle from the bf16 inputs, with the tolerance of every other parity test
        gA = float(g_a.item()) if g_a is not None else 1.0
        gW = float(g_w.item()) if g_w is not None else 1.0
        Aq, Asf = oracle_quantize(A.cpu(), fmt, "ceil", gA)
        bits = torch.int32 if out_dtype == torch.float32 else torch.int16
        assert torch.equal(out.view(bits), expect.view(bits)), "noalloc differs from mxq_linear at M=%d" % M
        ref, abs_sum = oracle.gemm(Aq, Asf, Wq_ref, Wsf_ref, M, N, K, FMTS[fmt], gA=gA, gB=gW)
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        if out_dtype == torch.float32:
            check_fp32(got, ref, abs_sum, "noalloc vs oracle M=%d" % M)
        else:
            check_bf16(got, ref, abs_sum, "noalloc vs oracle M=%d" % M)


def test_noalloc_rejects_problems_beyond_its_scratch():
    M, N, K = 8192, 256, 5120  # needs 21.0 MB + 1.3 MB of workspace, more than the 8 MiB array
    assert mxq.mxq_linear_workspace_size(M, K, mxq.MXFP4) > (8 << 20)
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    Wq = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    Wsf = torch.empty(mxq.sf_bytes(N, K, "mxfp4"), dtype=torch.uint8, device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(x, Wq, Wsf, N, "mxfp4", "ceil", out) == -5  # MXQ_ERR_WORKSPACE, nothing launched


def test_noalloc_error_codes_match_linear():
    """Bad arguments give mxq_linear's codes, in its order, before anything is launched or looked
    up: an unknown format is MXQ_ERR_UNSUPPORTED (not a shape error)."""
    P = 0x10000  # never dereferenced: every case fails validation first
    L = mxq.lib()
    assert L.mxq_linear_noalloc(P, P, P, None, None, 4, 4, 128, 7, 1, 0, P, None) == -4
    assert L.mxq_linear_noalloc(P, P, P, None, None, 4, 4, 128, 0, 9, 0, P, None) == -4
    assert L.mxq_linear_noalloc(None, P, P, None, None, 4, 4, 128, 0, 1, 0, P, None) == -1
    assert L.mxq_linear_noalloc(P, P, P, None, None, 4, 4, 96, 0, 1, 0, P, None) == -2
    assert L.mxq_linear_noalloc(P + 8, P, P, None, None, 4, 4, 128, 0, 1, 0, P, None) == -3
