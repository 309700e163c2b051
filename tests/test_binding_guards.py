"""CPU checks of the Python binding's host-side guards: before a tensor's pointer crosses the C
ABI (which sees no sizes), the binding refuses wrong element types and buffers smaller than the
call reads or writes.  The compute entry points are replaced by a stand-in that records the call;
the size helpers are the library's own."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_mx_b200 import build as mxq_build
from nvfp4_block_scaled_mx_b200 import mxq

COMPUTE = {"mxq_quantize", "mxq_quantize_running", "mxq_fake_quantize", "mxq_swizzle_scales", "mxq_global_scale",
           "mxq_gemm", "mxq_gemm_w4a16", "mxq_linear"}


class _Recorder:
    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in COMPUTE:
            def stub(*args):
                self.calls.append(name)
                return 0
            return stub
        return getattr(self.real, name)


@pytest.fixture()
def rec(monkeypatch):
    mxq_build.build()
    r = _Recorder(mxq.lib())
    monkeypatch.setattr(mxq, "lib", lambda: r)
    monkeypatch.setattr(mxq, "_ptr", lambda t: None if t is None else 0)
    monkeypatch.setattr(mxq, "_stream", lambda stream=None: None)
    return r


def _bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def _u8(n):
    return torch.zeros(n, dtype=torch.uint8)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("M,K", [(130, 1056), (1, 256), (3, 64)])
def test_quantize_sizes(rec, fmt, M, K):
    bs = 16 if fmt == "nvfp4" else 32
    if K % bs:
        pytest.skip("K not a multiple of the block")
    g = torch.ones(1, dtype=torch.float32) if fmt == "nvfp4" else None
    q, sf = mxq.quantize(_bf16(M, K), fmt, "ceil", global_scale=g)
    qn = M * (K if fmt == "mxfp8" else K // 2)
    assert q.numel() == qn and sf.numel() == mxq.sf_bytes(M, K, fmt)
    # caller-owned buffers of exactly the right size, both layouts
    mxq.quantize(_bf16(M, K), fmt, "ceil", global_scale=g, q_out=_u8(qn), sf_out=_u8(mxq.sf_bytes(M, K, fmt)))
    mxq.quantize(_bf16(M, K), fmt, "ceil", global_scale=g, layout=mxq.SF_ROWMAJOR, q_out=_u8(qn),
                 sf_out=_u8(M * K // bs))
    assert rec.calls == ["mxq_quantize"] * 3
    with pytest.raises(ValueError, match="q_out"):
        mxq.quantize(_bf16(M, K), fmt, "ceil", global_scale=g, q_out=_u8(qn - 1))
    with pytest.raises(ValueError, match="sf_out"):
        mxq.quantize(_bf16(M, K), fmt, "ceil", global_scale=g, sf_out=_u8(mxq.sf_bytes(M, K, fmt) - 1))
    with pytest.raises(ValueError, match="bfloat16"):
        mxq.quantize(torch.zeros(M, K), fmt, "ceil", global_scale=g)
    assert rec.calls == ["mxq_quantize"] * 3  # nothing reached the library


def test_global_scale_and_fake_and_running(rec):
    x = _bf16(37, 320)
    mxq.global_scale(x)
    mxq.fake_quantize(x, "mxfp4", "ceil", out=x)  # in place
    g = torch.ones(1, dtype=torch.float32)
    mxq.quantize_running(x, g, torch.empty(1, dtype=torch.float32))
    assert rec.calls == ["mxq_global_scale", "mxq_fake_quantize", "mxq_quantize_running"]
    with pytest.raises(ValueError, match="out"):
        mxq.fake_quantize(x, "mxfp4", "ceil", out=torch.zeros(37, 320, dtype=torch.float16))
    with pytest.raises(ValueError, match="global_scale"):
        mxq.fake_quantize(x, "nvfp4", "even", global_scale=torch.ones(1, dtype=torch.float64))
    with pytest.raises(ValueError, match="amax_out"):
        mxq.quantize_running(x, g, torch.empty(0, dtype=torch.float32))
    with pytest.raises(ValueError, match="x"):
        mxq.global_scale(torch.zeros(8, dtype=torch.float32))
    with pytest.raises(ValueError, match="2-D"):
        mxq.quantize(_bf16(4, 8, 32), "mxfp4")


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
def test_gemm_linear_w4a16_sizes(rec, fmt):
    M, N, K = 200, 333, 1024
    bs = 16 if fmt == "nvfp4" else 32
    qa = M * (K if fmt == "mxfp8" else K // 2)
    qb = N * (K if fmt == "mxfp8" else K // 2)
    # scales as the oracle swizzles them (what the parity tests hand in)
    A_sf = torch.from_numpy(oracle.swizzle(np.zeros((M, K // bs), np.uint8)))
    B_sf = torch.from_numpy(oracle.swizzle(np.zeros((N, K // bs), np.uint8)))
    g = torch.ones(1, dtype=torch.float32) if fmt == "nvfp4" else None
    for out_dtype in (torch.float32, torch.bfloat16):
        out = mxq.gemm(_u8(qa), A_sf, _u8(qb), B_sf, M, N, K, fmt, out_dtype=out_dtype, g_A=g, g_B=g)
        assert out.dtype == out_dtype and out.shape == (M, N)
        mxq.linear(_bf16(M, K), _u8(qb), B_sf, N, fmt, out_dtype=out_dtype, g_W=g, g_A=g)
    if fmt != "mxfp8":
        mxq.gemm_w4a16(_bf16(M, K), _u8(qb), B_sf, N, fmt, g_W=g)
    with pytest.raises(ValueError, match="B_sf"):
        mxq.gemm(_u8(qa), A_sf, _u8(qb), B_sf[:-1], M, N, K, fmt, g_A=g, g_B=g)
    with pytest.raises(ValueError, match="A_q"):
        mxq.gemm(_u8(qa - 16), A_sf, _u8(qb), B_sf, M, N, K, fmt, g_A=g, g_B=g)
    with pytest.raises(ValueError, match="out"):
        mxq.gemm(_u8(qa), A_sf, _u8(qb), B_sf, M, N, K, fmt, g_A=g, g_B=g,
                 out=torch.empty(M, N, dtype=torch.float32))  # bf16 requested
    with pytest.raises(ValueError, match="W_q"):
        mxq.linear(_bf16(M, K), _u8(qb // 2), B_sf, N, fmt, g_W=g, g_A=g)
    with pytest.raises(ValueError, match="out"):
        mxq.linear(_bf16(M, K), _u8(qb), B_sf, N, fmt, g_W=g, g_A=g, out=_bf16(M, N - 1))
    calls = ["mxq_gemm", "mxq_linear"] * 2 + ([] if fmt == "mxfp8" else ["mxq_gemm_w4a16"])
    assert rec.calls == calls


def test_swizzle_scales_sizes(rec):
    sf = torch.zeros(300, 160, dtype=torch.uint8)
    out = mxq.swizzle_scales(sf)
    assert out.numel() == 384 * 160
    with pytest.raises(ValueError, match="out"):
        mxq.swizzle_scales(sf, out=_u8(300 * 160))
    with pytest.raises(ValueError, match="sf_rowmajor"):
        mxq.swizzle_scales(torch.zeros(300, 160, dtype=torch.int32))
    assert rec.calls == ["mxq_swizzle_scales"]


def test_guard_errors_are_library_errors_too(rec):
    # callers that catch the library's errors also catch the guards', which carry the shape code
    with pytest.raises(mxq.MxqError) as e:
        mxq.quantize(_bf16(4, 64), "mxfp4", q_out=_u8(1))
    assert e.value.code == mxq.ERR_SHAPE and isinstance(e.value, ValueError)
    # a W4A16 call with FP8 weights reaches the library, which names the format
    Wq, Wsf = _u8(8 * 32), _u8(mxq.sf_bytes(8, 64, "mxfp4"))
    mxq.gemm_w4a16(_bf16(4, 64), Wq, Wsf, 8, "mxfp8")
    assert rec.calls == ["mxq_gemm_w4a16"]
    # K = 96 against buffers sized for K = 64: refused on the host
    with pytest.raises(mxq.MxqError):
        mxq.gemm_w4a16(_bf16(4, 96), Wq, Wsf, 8, "mxfp4")
