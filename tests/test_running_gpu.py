"""GPU parity of the NVFP4 running-max observer quantizer (mxq_quantize_running) against the
oracle over a sequence of batches: codes, scales and the running state must match exactly."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import mxq, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [mxq.SF_ROWMAJOR, mxq.SF_SWIZZLED])
@pytest.mark.parametrize("M,K", [(200, 1024), (3, 48)])
def test_running_max_sequence(layout, M, K):
    state = [torch.tensor([0.75], dtype=torch.float32, device="cuda"), torch.empty(1, dtype=torch.float32, device="cuda")]
    ref_state = np.float32(0.75)
    for step, scale in enumerate([1.0, 3.0, 0.5, 8.0]):
        x = (synth.random_bf16((M, K), 40 + step).float() * scale).to(torch.bfloat16)
        q, sf = mxq.quantize_running(x.cuda(), state[0], state[1], layout=layout)
        torch.cuda.synchronize()
        q_ref, sf_ref, new_ref = oracle.quantize_running(x, ref_state)
        assert np.array_equal(q.cpu().numpy(), q_ref)
        sf_gpu = sf.cpu().numpy()
        if layout == mxq.SF_SWIZZLED:
            assert np.array_equal(sf_gpu, oracle.swizzle(sf_ref))
        else:
            assert np.array_equal(sf_gpu.reshape(sf_ref.shape), sf_ref)
        assert state[1].item() == new_ref
        assert state[0].item() == ref_state  # the input state is read-only
        ref_state = new_ref
        state.reverse()


def test_running_rejects_aliased_state():
    x = torch.ones(4, 32, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(mxq.MxqError):
        mxq.quantize_running(x, s, s)
