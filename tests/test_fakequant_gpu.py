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
