"""Thin ctypes binding of libmxq.so (the C ABI in include/mxq.h).

The raw functions keep the C names and arguments (pointers as ints, sizes, enums, a stream
handle).  The tensor helpers below only allocate outputs with torch and marshal arguments; every
step of the computation runs in the library's kernels.  There is no fallback: if the library is
missing or the device is not an sm_100 part, the calls raise.
"""
import ctypes
import os

import torch

MXFP4, NVFP4, MXFP8 = 0, 1, 2
EVEN, CEIL = 0, 1
OUT_BF16, OUT_FP32 = 0, 1
SF_ROWMAJOR, SF_SWIZZLED = 0, 1

FMT = {"mxfp4": MXFP4, "nvfp4": NVFP4, "mxfp8": MXFP8}
RULE = {"even": EVEN, "ceil": CEIL}

ERR_SHAPE = -2
ERR_TIMEOUT = -7

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxq.so")

# name -> (restype, argtypes)
_P, _I64, _I, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "mxq_block_size": (_I, [_I]),
    "mxq_q_bytes": (_I, [_I64, _I64, _I, ctypes.POINTER(_SZ)]),
    "mxq_sf_bytes": (_I, [_I64, _I64, _I, _I, ctypes.POINTER(_SZ)]),
    "mxq_quantize": (_I, [_P, _I64, _I64, _I, _I, _P, _P, _P, _I, _P]),
    "mxq_quantize_running": (_I, [_P, _I64, _I64, _P, _P, _P, _P, _I, _P]),
    "mxq_fake_quantize": (_I, [_P, _I64, _I64, _I, _I, _P, _P, _P]),
    "mxq_swizzle_scales": (_I, [_P, _I64, _I64, _P, _P]),
    "mxq_global_scale": (_I, [_P, _I64, _P, _P, _P]),
    "mxq_amax": (_I, [_P, _I64, _P, _P]),
    "mxq_gemm": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _P, _P]),
    "mxq_gemm_w4a16": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _P, _P]),
    "mxq_linear_workspace_size": (_SZ, [_I64, _I64, _I]),
    "mxq_linear_kernel_count": (_I, [_I64, _I64, _I64, _I]),
    "mxq_linear": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _P, _SZ, _P, _P]),
    "mxq_linear_noalloc": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _I, _I, _P, _P]),
    "mxq_device_status": (_I, [ctypes.POINTER(_I), _I, _P]),
    "mxq_selftest_timeout": (_I, [_U64, _P]),
    "mxq_strerror": (ctypes.c_char_p, [_I]),
}

_lib = None


class MxqError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, lib().mxq_strerror(code).decode(), code))


class MxqBufferError(MxqError, ValueError):
    """A tensor handed to the binding does not fit the call (element type, rank or size); raised
    before anything reaches the library, with the shape error code."""

    def __init__(self, msg):
        self.code = ERR_SHAPE
        Exception.__init__(self, msg)


def lib():
    """Load libmxq.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError("libmxq.so not built: run `python -m nvfp4_block_scaled_mx_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(rc, where):
    if rc != 0:
        raise MxqError(rc, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("mxq works on CUDA tensors only (got a %s tensor)" % t.device)
    if not t.is_contiguous():
        raise ValueError("mxq needs contiguous tensors")
    return t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _fmt(f):
    return FMT[f] if isinstance(f, str) else int(f)


def _rule(r):
    return RULE[r] if isinstance(r, str) else int(r)


# ---------------------------------------------------------------- raw C entry points (same names)

def mxq_quantize(x, M, K, fmt, rule, global_scale, q_out, sf_out, layout, stream):
    return lib().mxq_quantize(x, M, K, fmt, rule, global_scale, q_out, sf_out, layout, stream)


def mxq_fake_quantize(x, M, K, fmt, rule, global_scale, y, stream):
    return lib().mxq_fake_quantize(x, M, K, fmt, rule, global_scale, y, stream)


def mxq_swizzle_scales(sf_rowmajor, rows, kblocks, sf_swizzled, stream):
    return lib().mxq_swizzle_scales(sf_rowmajor, rows, kblocks, sf_swizzled, stream)


def mxq_global_scale(x, n, g_out, amax_out, stream):
    return lib().mxq_global_scale(x, n, g_out, amax_out, stream)


def mxq_amax(x, n, amax_out, stream):
    return lib().mxq_amax(x, n, amax_out, stream)


def mxq_gemm(A_q, A_sf, B_q, B_sf, g_A, g_B, M, N, K, fmt, out_type, out, stream):
    return lib().mxq_gemm(A_q, A_sf, B_q, B_sf, g_A, g_B, M, N, K, fmt, out_type, out, stream)


def mxq_gemm_w4a16(A, W_q, W_sf, g_W, M, N, K, fmt, out_type, out, stream):
    return lib().mxq_gemm_w4a16(A, W_q, W_sf, g_W, M, N, K, fmt, out_type, out, stream)


def mxq_linear(x, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, workspace, ws_bytes, out, stream):
    return lib().mxq_linear(x, W_q, W_sf, g_W, g_A, M, N, K, fmt, act_rule, out_type, workspace, ws_bytes, out,
                            stream)


def mxq_linear_workspace_size(M, K, fmt):
    return lib().mxq_linear_workspace_size(M, K, fmt)


def linear_kernel_count(M, N, K, fmt):
    """Kernels one linear() call launches for this problem on the current device (1 or 2)."""
    n = lib().mxq_linear_kernel_count(M, N, K, _fmt(fmt))
    _check(n if n < 0 else 0, "mxq_linear_kernel_count")
    return n


def mxq_device_status(reset=True, stream=None):
    v = ctypes.c_int(0)
    _check(lib().mxq_device_status(ctypes.byref(v), 1 if reset else 0, _stream(stream)), "mxq_device_status")
    return v.value


def mxq_selftest_timeout(timeout_ns, stream=None):
    _check(lib().mxq_selftest_timeout(int(timeout_ns), _stream(stream)), "mxq_selftest_timeout")


# ---------------------------------------------------------------- tensor helpers

def block_size(fmt):
    return 16 if _fmt(fmt) == NVFP4 else 32


def q_shape(rows, K, fmt):
    return (rows, K if _fmt(fmt) == MXFP8 else K // 2)


def sf_bytes(rows, K, fmt, layout=SF_SWIZZLED):
    n = ctypes.c_size_t(0)
    _check(lib().mxq_sf_bytes(rows, K, _fmt(fmt), layout, ctypes.byref(n)), "mxq_sf_bytes")
    return n.value


def _q_bytes(rows, K, f):
    return rows * (K if f == MXFP8 else K // 2)


def _need(t, name, nbytes, dtype=None):
    """Host-side guard before a tensor's pointer crosses the C ABI, which sees no sizes: the kernels
    read or write `nbytes` through it, so a smaller buffer, or one of another element type where
    the element type matters, is refused here instead of being overrun on the device."""
    if t is None:
        return
    if dtype is not None and t.dtype != dtype:
        raise MxqBufferError("%s must be %s (got %s)" % (name, dtype, t.dtype))
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise MxqBufferError("%s holds %d bytes, the call needs %d" % (name, have, nbytes))


def _need_x(x, name="x"):
    if x.dim() != 2:
        raise MxqBufferError("%s must be a 2-D [M, K] tensor (got %d dims)" % (name, x.dim()))
    _need(x, name, 2 * x.numel(), torch.bfloat16)


def quantize(x, fmt, rule=EVEN, global_scale=None, layout=SF_SWIZZLED, q_out=None, sf_out=None, stream=None):
    """x [M, K] bf16 (CUDA) -> (q uint8 [M, K/2] or [M, K], sf uint8 flat (swizzled) or [M, K/bs])."""
    f, r = _fmt(fmt), _rule(rule)
    _need_x(x)
    M, K = x.shape
    if q_out is None:
        q_out = torch.empty(q_shape(M, K, f), dtype=torch.uint8, device=x.device)
    if sf_out is None:
        if layout == SF_SWIZZLED:
            sf_out = torch.empty(sf_bytes(M, K, f, layout), dtype=torch.uint8, device=x.device)
        else:
            sf_out = torch.empty((M, K // block_size(f)), dtype=torch.uint8, device=x.device)
    _need(q_out, "q_out", _q_bytes(M, K, f))
    _need(sf_out, "sf_out", sf_bytes(M, K, f, layout))
    _need(global_scale, "global_scale", 4, torch.float32)
    _check(mxq_quantize(_ptr(x), M, K, f, r, _ptr(global_scale), _ptr(q_out), _ptr(sf_out), layout,
                        _stream(stream)), "mxq_quantize")
    return q_out, sf_out


def quantize_running(x, amax_in, amax_out, layout=SF_SWIZZLED, q_out=None, sf_out=None, stream=None):
    """NVFP4 quantize of x with g = amax_in/2688; amax_out <- max(amax_in, max|x|)."""
    _need_x(x)
    M, K = x.shape
    if q_out is None:
        q_out = torch.empty(q_shape(M, K, NVFP4), dtype=torch.uint8, device=x.device)
    if sf_out is None:
        if layout == SF_SWIZZLED:
            sf_out = torch.empty(sf_bytes(M, K, NVFP4, layout), dtype=torch.uint8, device=x.device)
        else:
            sf_out = torch.empty((M, K // 16), dtype=torch.uint8, device=x.device)
    _need(q_out, "q_out", _q_bytes(M, K, NVFP4))
    _need(sf_out, "sf_out", sf_bytes(M, K, NVFP4, layout))
    _need(amax_in, "amax_in", 4, torch.float32)
    _need(amax_out, "amax_out", 4, torch.float32)
    _check(lib().mxq_quantize_running(_ptr(x), M, K, _ptr(amax_in), _ptr(amax_out), _ptr(q_out), _ptr(sf_out), layout,
                                      _stream(stream)), "mxq_quantize_running")
    return q_out, sf_out


def fake_quantize(x, fmt, rule=EVEN, global_scale=None, out=None, stream=None):
    """x [M, K] bf16 (CUDA) -> bf16 quantize-dequantize of x (out may be x for in-place)."""
    _need_x(x)
    M, K = x.shape
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", 2 * M * K, torch.bfloat16)
    _need(global_scale, "global_scale", 4, torch.float32)
    _check(mxq_fake_quantize(_ptr(x), M, K, _fmt(fmt), _rule(rule), _ptr(global_scale), _ptr(out), _stream(stream)),
           "mxq_fake_quantize")
    return out


def swizzle_scales(sf_rowmajor, out=None, stream=None):
    rows, kb = sf_rowmajor.shape
    n = ((rows + 127) // 128) * 128 * ((kb + 3) // 4) * 4
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=sf_rowmajor.device)
    _need(sf_rowmajor, "sf_rowmajor", rows * kb, torch.uint8)
    _need(out, "out", n)
    _check(mxq_swizzle_scales(_ptr(sf_rowmajor), rows, kb, _ptr(out), _stream(stream)), "mxq_swizzle_scales")
    return out


def global_scale(x, stream=None):
    """NVFP4 decode-direction global scale g = amax / 2688 and amax, as device fp32[1] tensors."""
    _need(x, "x", 2 * x.numel(), torch.bfloat16)
    g = torch.empty(1, dtype=torch.float32, device=x.device)
    amax = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(mxq_global_scale(_ptr(x), x.numel(), _ptr(g), _ptr(amax), _stream(stream)), "mxq_global_scale")
    return g, amax


def amax(x, stream=None):
    """max |x| over the whole tensor, as a device fp32[1] tensor."""
    _need(x, "x", 2 * x.numel(), torch.bfloat16)
    out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(mxq_amax(_ptr(x), x.numel(), _ptr(out), _stream(stream)), "mxq_amax")
    return out


def gemm(A_q, A_sf, B_q, B_sf, M, N, K, fmt, out_dtype=torch.bfloat16, g_A=None, g_B=None, out=None, stream=None):
    f = _fmt(fmt)
    ot = OUT_FP32 if out_dtype == torch.float32 else OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A_q.device)
    _need(A_q, "A_q", _q_bytes(M, K, f))
    _need(B_q, "B_q", _q_bytes(N, K, f))
    _need(A_sf, "A_sf", sf_bytes(M, K, f))
    _need(B_sf, "B_sf", sf_bytes(N, K, f))
    _need(g_A, "g_A", 4, torch.float32)
    _need(g_B, "g_B", 4, torch.float32)
    _need(out, "out", M * N * (4 if ot == OUT_FP32 else 2), torch.float32 if ot == OUT_FP32 else torch.bfloat16)
    _check(mxq_gemm(_ptr(A_q), _ptr(A_sf), _ptr(B_q), _ptr(B_sf), _ptr(g_A), _ptr(g_B), M, N, K, f, ot, _ptr(out),
                    _stream(stream)), "mxq_gemm")
    return out


def gemm_w4a16(A, W_q, W_sf, N, fmt, g_W=None, out_dtype=torch.bfloat16, out=None, stream=None):
    """Weight-only GEMM: out = A dq(W)^T with A [M, K] bf16 and W pre-quantized (swizzled scales)."""
    f = _fmt(fmt)
    _need_x(A, "A")
    M, K = A.shape
    ot = OUT_FP32 if out_dtype == torch.float32 else OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=A.device)
    if f == MXFP8:  # 4-bit weights only: the library rejects the format before any launch
        _check(mxq_gemm_w4a16(_ptr(A), _ptr(W_q), _ptr(W_sf), _ptr(g_W), M, N, K, f, ot, _ptr(out), _stream(stream)),
               "mxq_gemm_w4a16")
        return out
    _need(W_q, "W_q", _q_bytes(N, K, f))
    _need(W_sf, "W_sf", sf_bytes(N, K, f))
    _need(g_W, "g_W", 4, torch.float32)
    _need(out, "out", M * N * (4 if ot == OUT_FP32 else 2), torch.float32 if ot == OUT_FP32 else torch.bfloat16)
    _check(mxq_gemm_w4a16(_ptr(A), _ptr(W_q), _ptr(W_sf), _ptr(g_W), M, N, K, f, ot, _ptr(out), _stream(stream)),
           "mxq_gemm_w4a16")
    return out


def linear(x, W_q, W_sf, N, fmt, act_rule=CEIL, out_dtype=torch.bfloat16, g_W=None, g_A=None, workspace=None,
           out=None, stream=None):
    """Quantize x per token, then out = A_q W_q^T (W pre-quantized with swizzled scales)."""
    f = _fmt(fmt)
    _need_x(x)
    M, K = x.shape
    ws = mxq_linear_workspace_size(M, K, f)
    if workspace is None:
        workspace = torch.empty(ws, dtype=torch.uint8, device=x.device)
    ot = OUT_FP32 if out_dtype == torch.float32 else OUT_BF16
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _need(W_q, "W_q", _q_bytes(N, K, f))
    _need(W_sf, "W_sf", sf_bytes(N, K, f))
    _need(g_W, "g_W", 4, torch.float32)
    _need(g_A, "g_A", 4, torch.float32)
    _need(out, "out", M * N * (4 if ot == OUT_FP32 else 2), torch.float32 if ot == OUT_FP32 else torch.bfloat16)
    _check(mxq_linear(_ptr(x), _ptr(W_q), _ptr(W_sf), _ptr(g_W), _ptr(g_A), M, N, K, f, _rule(act_rule), ot,
                      _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
           "mxq_linear")
    return out
