"""GPU parity of mxq_quantize / mxq_swizzle_scales / mxq_global_scale against the CPU oracle:
quantized bytes and scales must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth
from tests.helpers import FMTS, RULES, oracle_quantize, to_np
from tests.test_oracle_quant import _adversarial_bf16

pytestmark = pytest.mark.gpu

COMBOS = [("mxfp4", "even"), ("mxfp4", "ceil"), ("mxfp8", "even"), ("mxfp8", "ceil"), ("nvfp4", "even")]


def _run(x_cpu, fmt, rule, layout, g=None):
    x = x_cpu.cuda()
    gd = None
    if fmt == "nvfp4":
        gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    q, sf = mxq.quantize(x, fmt, rule, global_scale=gd, layout=layout)
    torch.cuda.synchronize()
    return to_np(q), to_np(sf)


@pytest.mark.parametrize("fmt,rule", COMBOS)
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (5, 80), (1, 32), (3, 64), (7, 128), (9, 384), (37, 320),
                                   (130, 1056), (256, 5120), (2053, 8192)])
def test_quantize_matches_oracle(fmt, rule, shape):
    """Shapes cover a single block, NVFP4 tensors whose last 16-element block is half a 32-element
    row of the input stream (M * K = 16 mod 32), partial 256-row input boxes, more boxes than CTAs
    (the input ring wraps), and rows whose block count is and is not a multiple of 4 (scale bytes
    gathered across lanes into 32-bit stores, or stored one by one)."""
    M, K = shape
    bs = 16 if fmt == "nvfp4" else 32
    if K % bs:
        pytest.skip("K not a multiple of the block")
    x = _adversarial_bf16(M, K, M * 7 + K, huge=3.0e38 if fmt != "nvfp4" else 3.0e6, bs=bs)
    g = 1.0
    if fmt == "nvfp4":
        g, _ = oracle.global_scale(x)
    q_ref, sf_ref = oracle_quantize(x, fmt, rule, g)
    for layout in (mxq.SF_ROWMAJOR, mxq.SF_SWIZZLED):
        q, sf = _run(x, fmt, rule, layout, float(g))
        assert np.array_equal(q, q_ref), "element codes differ (%s/%s %s)" % (fmt, rule, shape)
        if layout == mxq.SF_ROWMAJOR:
            assert np.array_equal(sf.reshape(sf_ref.shape), sf_ref)
        else:
            assert np.array_equal(sf, oracle.swizzle(sf_ref)), "swizzled scales (incl. zero padding) differ"


@pytest.mark.parametrize("g", ["tensor", 1.0, 2.0 ** -20, 3.7e-3, 1.0e4, 2.0 ** -100, 2.0 ** 100, 2.0 ** -140,
                               1.0e-40])
def test_nvfp4_every_block_amax(g):
    """Every positive finite bf16 value is the amax of one 16-element NVFP4 block (its other
    elements are seeded fractions of it, both signs), so the scale sequence t = fl(amax / 6),
    u = fl(t / g) runs over every block amax the format can meet: scales and codes must equal the
    oracle's IEEE fp32 arithmetic bit for bit, for the tensor's own global scale and for fixed ones
    that send most scales to 0, saturate them at 448, make t and u subnormal, or make g subnormal
    (where fl(1/d) overflows to +inf for the large scales)."""
    pats = np.arange(1, 0x7F80, dtype=np.uint16)  # 0x0001 .. 0x7F7F: every positive finite bf16
    nb, K = pats.size, 256
    rows = (nb * 16 + K - 1) // K
    amax = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).float()
    frac = torch.from_numpy(np.random.default_rng(5).uniform(-1.0, 1.0, size=(nb, 16))).float()
    frac[:, 0], frac[:, 1] = 1.0, -1.0
    blocks = (amax[:, None] * frac).to(torch.bfloat16).reshape(-1)
    x = torch.zeros(rows * K, dtype=torch.bfloat16)
    x[: blocks.numel()] = blocks
    x = x.reshape(rows, K)
    gv = oracle.global_scale(x)[0] if g == "tensor" else float(g)
    q_ref, sf_ref = oracle_quantize(x, "nvfp4", "even", gv)
    q, sf = _run(x, "nvfp4", "even", mxq.SF_ROWMAJOR, float(gv))
    assert np.array_equal(sf.reshape(sf_ref.shape), sf_ref), "scales differ (g = %r)" % (gv,)
    assert np.array_equal(q, q_ref), "codes differ (g = %r)" % (gv,)


@pytest.mark.parametrize("fmt,rule", COMBOS)
def test_quantize_random_fuzz(fmt, rule):
    """Seeded fuzz over plain Gaussian data with per-row dynamic range, many blocks."""
    g = torch.Generator().manual_seed(11)
    mism = 0
    total = 0
    for it in range(6):
        M = int(torch.randint(1, 300, (1,), generator=g))
        K = 64 * int(torch.randint(1, 40, (1,), generator=g))
        x = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(M, 1, generator=g) * 4)).to(torch.bfloat16)
        gs = 1.0
        if fmt == "nvfp4":
            gs, _ = oracle.global_scale(x)
        q_ref, sf_ref = oracle_quantize(x, fmt, rule, gs)
        q, sf = _run(x, fmt, rule, mxq.SF_ROWMAJOR, float(gs))
        mism += int((q != q_ref).sum()) + int((sf.reshape(sf_ref.shape) != sf_ref).sum())
        total += q.size + sf.size
    assert mism == 0, "%d / %d mismatching bytes" % (mism, total)


def test_swizzle_kernel_matches_oracle():
    for rows, kb in [(1, 1), (5, 3), (128, 4), (300, 160), (257, 1088)]:
        sf = torch.randint(0, 256, (rows, kb), dtype=torch.uint8, generator=torch.Generator().manual_seed(rows))
        out = mxq.swizzle_scales(sf.cuda())
        torch.cuda.synchronize()
        assert np.array_equal(to_np(out), oracle.swizzle(sf.numpy()))


def test_global_scale_matches_oracle():
    for n, seed in [(16, 1), (1000, 2), (8192 * 17 + 5, 3)]:
        x = synth.random_bf16((n,), seed, std=3.0)
        g_ref, amax_ref = oracle.global_scale(x)
        g, amax = mxq.global_scale(x.cuda())
        torch.cuda.synchronize()
        assert to_np(amax)[0] == amax_ref and to_np(g)[0] == g_ref
