"""Pins of the oracle's weight-only (W4A16) GEMM: bf16 activations times dequantized MXFP4 / NVFP4
weights, the serving mode of the NVFP4 weight-only checkpoint and the Marlin mode of the MXFP4
checkpoints.

A slip in the oracle (transposed operand, dropped global scale, A read as quantized codes, wrong
block index) fails at least one check:
  - numpy fp64 matmul of ml_dtypes-decoded weights and torch-decoded bf16 activations;
  - bit equality with the already pinned W4A4 GEMM when the bf16 activations are exactly the
    dequantized values of quantized activations;
  - exact integer arithmetic with unit scales.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_mx_b200 import synth
from tests.test_oracle_quant import _lib_dequant


def _f64(t):
    return t.float().double().numpy()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_w4a16_matches_numpy_fp64(orc, fmt):
    f = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4}[fmt]
    M, N, K = 7, 11, 256
    A = synth.random_bf16((M, K), 31, std=1.5)
    W = synth.random_bf16((N, K), 32, std=0.02)
    gW = 1.0
    if fmt == "nvfp4":
        gW, _ = orc.global_scale(W)
    Wq, Wsf = orc.quantize(W, f, orc.EVEN, g=float(gW))
    out, absout = orc.gemm_w4a16(A, Wq, Wsf, M, N, K, f, gB=float(gW))
    a = _f64(A)
    b = _lib_dequant(Wq, Wsf, K, fmt, float(gW))
    ref = a @ b.T
    assert np.all(np.abs(out - ref) <= 1e-13 * absout)
    assert np.allclose(absout, np.abs(a) @ np.abs(b).T, rtol=1e-12)
    rows, cols = np.array([6, 0, 2]), np.array([10, 3, 4])
    sub, _ = orc.gemm_w4a16(A, Wq, Wsf, M, N, K, f, gB=float(gW), rows=rows, cols=cols)
    assert np.array_equal(sub, out[np.ix_(rows, cols)])


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_w4a16_equals_w4a4_on_representable_activations(orc, fmt):
    """With bf16 activations equal to dq(A_q) the weight-only product is the W4A4 product, term by
    term in the same order, so the two oracle functions agree bit for bit."""
    f = {"mxfp4": orc.MXFP4, "nvfp4": orc.NVFP4}[fmt]
    M, N, K = 5, 9, 320
    A = synth.random_bf16((M, K), 41)
    W = synth.random_bf16((N, K), 42, std=0.02)
    gW = 1.0
    if fmt == "nvfp4":
        gW, _ = orc.global_scale(W)
    Aq, Asf = orc.quantize(A, f, orc.CEIL, g=1.0)
    Wq, Wsf = orc.quantize(W, f, orc.EVEN, g=float(gW))
    a_vals = orc.dequantize(Aq, Asf, K, f, g=1.0)
    A_rep = torch.from_numpy(a_vals).to(torch.bfloat16)
    assert np.array_equal(_f64(A_rep), a_vals)  # exactly representable in bf16
    w16, _ = orc.gemm_w4a16(A_rep, Wq, Wsf, M, N, K, f, gB=float(gW))
    w44, _ = orc.gemm(Aq, Asf, Wq, Wsf, M, N, K, f, gA=1.0, gB=float(gW))
    assert np.array_equal(w16, w44)


def test_w4a16_exact_integers(orc):
    # unit E8M0 scales and E2M1 codes: 2*w is an integer; small integer activations are exact in
    # bf16, so every partial sum is an exact integer / 2 in fp64
    rng = np.random.default_rng(9)
    M, N, K = 3, 5, 96
    a_int = rng.integers(-20, 21, (M, K))
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    sfb = np.full((N, K // 32), 127, np.uint8)
    A = torch.from_numpy(a_int.astype(np.float32)).to(torch.bfloat16)
    out, _ = orc.gemm_w4a16(A, pack(cb), sfb, M, N, K, orc.MXFP4)
    twice = np.array([0, 1, 2, 3, 4, 6, 8, 12], np.int64)
    ib = twice[cb & 7] * np.where(cb & 8, -1, 1)
    assert np.array_equal(out * 2, (a_int @ ib.T).astype(np.float64))
    # a scale of 2^-2 on one block of weight row 4 scales exactly that block's contribution
    sfb2 = sfb.copy()
    sfb2[4, 2] = 125
    out2, _ = orc.gemm_w4a16(A, pack(cb), sfb2, M, N, K, orc.MXFP4)
    part = (a_int[:, 64:96] @ ib[4, 64:96]).astype(np.float64) / 2
    assert np.array_equal(out[:, 4] - out2[:, 4], 0.75 * part)
    assert np.array_equal(np.delete(out2, 4, axis=1), np.delete(out, 4, axis=1))
