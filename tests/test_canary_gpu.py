"""Out-of-bounds writes, checked with canaries (a stand-in for a memory-checking tool, which these
tests do not run): every output buffer of a call sits inside a larger allocation, 4 KB from its start
(keeping 16-byte alignment), whose bytes outside the buffer hold a sentinel pattern; after the call,
not one of them may have changed.  Shapes are those of the parity tests: ragged M, N and K tails, a
single element, several tiles, and both the one-launch and the two-launch linear paths."""
import pytest
import torch

from nvfp4_block_scaled_mx_b200 import mxq, synth

pytestmark = pytest.mark.gpu

PAD = 4096  # bytes of canary on each side


class Canary:
    """A view of `nbytes` bytes (as `dtype`, shaped `shape`) inside a sentinel-filled allocation."""

    def __init__(self, nbytes, dtype=torch.uint8, shape=None, device="cuda"):
        self.buf = torch.full((PAD + nbytes + PAD,), 0xA5, dtype=torch.uint8, device=device)
        self.nbytes = nbytes
        view = self.buf[PAD:PAD + nbytes].view(dtype)
        self.t = view.view(shape) if shape is not None else view

    def intact(self):
        b = self.buf.cpu()
        return bool((b[:PAD] == 0xA5).all()) and bool((b[PAD + self.nbytes:] == 0xA5).all())


def _qbytes(M, K, fmt):
    return M * (K if fmt == "mxfp8" else K // 2)


@pytest.mark.parametrize("fmt,rule", [("mxfp4", "ceil"), ("mxfp4", "even"), ("nvfp4", "even"), ("mxfp8", "ceil")])
@pytest.mark.parametrize("M,K", [(1, 32), (37, 320), (130, 1056), (256, 5120)])
def test_quantize_and_fake_quantize_write_inside_their_buffers(fmt, rule, M, K):
    x = synth.random_bf16((M, K), M + K, device="cuda")
    g = mxq.global_scale(x)[0] if fmt == "nvfp4" else None
    for layout in (mxq.SF_ROWMAJOR, mxq.SF_SWIZZLED):
        q = Canary(_qbytes(M, K, fmt))
        sf = Canary(mxq.sf_bytes(M, K, fmt, layout))
        mxq.quantize(x, fmt, rule, global_scale=g, layout=layout, q_out=q.t, sf_out=sf.t)
        torch.cuda.synchronize()
        assert q.intact(), "codes written outside their buffer"
        assert sf.intact(), "scales written outside their buffer (layout %d)" % layout
        ref_q, ref_sf = mxq.quantize(x, fmt, rule, global_scale=g, layout=layout)
        assert torch.equal(q.t, ref_q.view(-1)) and torch.equal(sf.t, ref_sf.view(-1))
    y = Canary(2 * M * K, torch.bfloat16, (M, K))
    mxq.fake_quantize(x, fmt, rule, global_scale=g, out=y.t)
    torch.cuda.synchronize()
    assert y.intact(), "fake-quantized values written outside their buffer"
    assert torch.equal(y.t, mxq.fake_quantize(x, fmt, rule, global_scale=g))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (17, 300, 320), (129, 520, 1024), (300, 257, 576)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_and_linear_write_inside_their_output(fmt, M, N, K, out_dtype):
    A = synth.random_bf16((M, K), 3 * M + K, device="cuda")
    W = synth.random_bf16((N, K), 5 * N + K, std=0.02, device="cuda")
    g_a = g_w = None
    if fmt == "nvfp4":
        g_a, g_w = mxq.global_scale(A)[0], mxq.global_scale(W)[0]
    Aq, Asf = mxq.quantize(A, fmt, "ceil", global_scale=g_a)
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    es = 4 if out_dtype == torch.float32 else 2
    o1 = Canary(M * N * es, out_dtype, (M, N))
    mxq.gemm(Aq, Asf, Wq, Wsf, M, N, K, fmt, out_dtype=out_dtype, g_A=g_a, g_B=g_w, out=o1.t)
    o2 = Canary(M * N * es, out_dtype, (M, N))
    mxq.linear(A, Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=out_dtype, g_W=g_w, g_A=g_a, out=o2.t)
    torch.cuda.synchronize()
    assert o1.intact(), "GEMM output written outside its buffer"
    assert o2.intact(), "linear output written outside its buffer"
    assert torch.equal(o1.t, o2.t)
    if fmt != "mxfp8":
        o3 = Canary(M * N * es, out_dtype, (M, N))
        mxq.gemm_w4a16(A, Wq, Wsf, N, fmt, g_W=g_w, out_dtype=out_dtype, out=o3.t)
        torch.cuda.synchronize()
        assert o3.intact(), "W4A16 output written outside its buffer"


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("M,N,K", [(17, 300, 320), (129, 520, 1024), (300, 257, 576)])
def test_noalloc_writes_inside_its_output(fmt, M, N, K):
    """The allocation-free linear entry point writes its quantized activations into a static array
    of the library, next to its other device globals; an overrun there would corrupt them unseen.
    Its output must stay inside its canaried buffer, the device status word must stay clean, and a
    regular mxq_linear afterwards must still give the same bytes."""
    A = synth.random_bf16((M, K), 7 * M + K, device="cuda")
    W = synth.random_bf16((N, K), 11 * N + K, std=0.02, device="cuda")
    g_a = g_w = None
    if fmt == "nvfp4":
        g_a, g_w = mxq.global_scale(A)[0], mxq.global_scale(W)[0]
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    mxq.mxq_device_status(reset=True)
    o = Canary(M * N * 2, torch.bfloat16, (M, N))
    p = lambda t: None if t is None else t.data_ptr()
    rc = mxq.lib().mxq_linear_noalloc(p(A), p(Wq), p(Wsf), p(g_w), p(g_a), M, N, K, mxq.FMT[fmt], mxq.CEIL,
                                      mxq.OUT_BF16, p(o.t), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert o.intact(), "no-alloc linear output written outside its buffer"
    assert mxq.mxq_device_status(reset=True) == 0
    expect = mxq.linear(A, Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=torch.bfloat16, g_W=g_w, g_A=g_a)
    torch.cuda.synchronize()
    assert torch.equal(o.t.view(torch.int16), expect.view(torch.int16))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "mxfp8"])
@pytest.mark.parametrize("M,N,K", [(33, 1, 64), (129, 96, 1024), (300, 17, 576)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_small_n_linear_writes_inside_its_output(fmt, M, N, K, out_dtype):
    """The small-N linear kernel (more than 32 tokens, N <= 128) stores row by row with N tails."""
    A = synth.random_bf16((M, K), 13 * M + K, device="cuda")
    W = synth.random_bf16((N, K), 17 * N + K, std=0.02, device="cuda")
    g_a = g_w = None
    if fmt == "nvfp4":
        g_a, g_w = mxq.global_scale(A)[0], mxq.global_scale(W)[0]
    Wq, Wsf = mxq.quantize(W, fmt, "even", global_scale=g_w)
    es = 4 if out_dtype == torch.float32 else 2
    o = Canary(M * N * es, out_dtype, (M, N))
    mxq.linear(A, Wq, Wsf, N, fmt, act_rule="ceil", out_dtype=out_dtype, g_W=g_w, g_A=g_a, out=o.t)
    torch.cuda.synchronize()
    assert o.intact(), "small-N linear output written outside its buffer"
    assert mxq.mxq_device_status(reset=True) == 0
