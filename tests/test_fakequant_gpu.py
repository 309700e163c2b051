"""GPU parity of mxq_fake_quantize (quantize-dequantize to bf16) against the oracle: every output
bf16 bit pattern must match."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth
from tests.helpers import FMTS, RULES
from tests.test_oracle_quant import _adversarial_bf16

pytestmark = pytest.mark.gpu

COMBOS = [("mxfp4", "even"), ("mxfp4", "ceil"), ("mxfp8", "even"), ("mxfp8", "ceil"), ("nvfp4", "even")]


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("fmt,rule", COMBOS)
@pytest.mark.parametrize("shape", [(1, 16), (3, 48), (1, 32), (37, 320), (130, 1056), (256, 5120)])
def test_fake_quantize_matches_oracle(fmt, rule, shape):
    M, K = shape
    bs = 16 if fmt == "nvfp4" else 32
    if K % bs:
        pytest.skip("K not a multiple of the block")
    x = _adversarial_bf16(M, K, 3 * M + K, huge=3.0e38 if fmt != "nvfp4" else 3.0e6, bs=bs)
    g = 1.0
    gd = None
    if fmt == "nvfp4":
        g, _ = oracle.global_scale(x)
        gd = torch.tensor([float(g)], dtype=torch.float32, device="cuda")
    ref = oracle.fake_quantize(x, FMTS[fmt], RULES[rule], g=float(g))
    xd = x.cuda()
    y = mxq.fake_quantize(xd, fmt, rule, global_scale=gd)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), ref)
    # in place
    mxq.fake_quantize(xd, fmt, rule, global_scale=gd, out=xd)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(xd), ref)


def test_fake_quantize_full_size_sampled_rows():
    A, _ = synth.make_inputs("prefill_gate_up", device="cuda", N=128)
    y = mxq.fake_quantize(A, "mxfp4", "ceil")
    torch.cuda.synchronize()
    rows = torch.unique(torch.randint(0, A.shape[0], (64,), generator=torch.Generator().manual_seed(5))).tolist()
    ref = oracle.fake_quantize(A[rows].cpu(), oracle.MXFP4, oracle.CEIL)
    assert np.array_equal(_bits(y[rows]), ref)


def _every_binade(bs, seed):
    """Two blocks per binade of the block amax, from below the smallest bf16 subnormal to the top of
    the bf16 range, one with an amax mantissa in [1, 1.4) and one in [1.6, 2) (so that CEIL moves up a
    binade in the second): every E8M0 scale code the MX formats can produce, and the clamp at 0."""
    g = np.random.default_rng(seed)
    ks = np.repeat(np.arange(-136, 128), 2)
    mant = np.where(np.arange(len(ks)) % 2 == 0, 1.0, 1.6) + g.uniform(0.0, 0.39, len(ks))
    blocks = g.uniform(-1.0, 1.0, (len(ks), bs)) * np.ldexp(1.0, ks)[:, None]
    blocks[:, 0] = np.ldexp(mant, ks) * g.choice([-1.0, 1.0], len(ks))
    return torch.from_numpy(blocks.reshape(-1, 128).astype(np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt,rule", COMBOS[:4])
def test_fake_quantize_every_scale_code(fmt, rule):
    # the MX decodes switch between a bf16 and an fp32 multiply by the scale code; both sides of
    # each switch point (and the ends of the exponent range) are in here
    x = _every_binade(32, 11)
    q, sf = oracle.quantize(x, FMTS[fmt], RULES[rule])
    switch_points = {0, 1, 2, 128, 129} if fmt == "mxfp4" else {0, 9, 10, 134, 135}
    assert switch_points <= set(np.unique(sf).tolist())
    ref = oracle.fake_quantize(x, FMTS[fmt], RULES[rule])
    y = mxq.fake_quantize(x.cuda(), fmt, rule)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), ref)


@pytest.mark.parametrize("g", [2.0 ** -140, 1.0e-30, 3.7e-6, 1.0, 1.0 / 2688, 5.0e20, 2.0 ** 100])
def test_fake_quantize_nvfp4_global_scales(g):
    x = _every_binade(16, 12)
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    ref = oracle.fake_quantize(x, oracle.NVFP4, oracle.EVEN, g=float(np.float32(g)))
    y = mxq.fake_quantize(x.cuda(), "nvfp4", "even", global_scale=gd)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(y), ref)
