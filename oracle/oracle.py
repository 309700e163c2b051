"""ctypes wrapper over the scalar C oracle (``mxq_oracle.c``).

Test infrastructure only: see the package docstring.  Arrays are numpy; bf16 tensors are passed
as their uint16 bit patterns.
"""
import ctypes
import os
import subprocess

import numpy as np

MXFP4, NVFP4, MXFP8 = 0, 1, 2
EVEN, CEIL = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mxq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force=False):
    """Compile the oracle with plain gcc (IEEE fp32/fp64, no contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        p, i64, i32, d, f = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
        L.orc_bf16_value.argtypes, L.orc_bf16_value.restype = [ctypes.c_uint16], d
        L.orc_e2m1_value.argtypes, L.orc_e2m1_value.restype = [ctypes.c_uint8], d
        L.orc_e2m1_encode.argtypes, L.orc_e2m1_encode.restype = [d], ctypes.c_uint8
        L.orc_e4m3_value.argtypes, L.orc_e4m3_value.restype = [ctypes.c_uint8], d
        L.orc_e4m3_encode.argtypes, L.orc_e4m3_encode.restype = [d], ctypes.c_uint8
        L.orc_e8m0_value.argtypes, L.orc_e8m0_value.restype = [ctypes.c_uint8], d
        L.orc_mx_exponent.argtypes, L.orc_mx_exponent.restype = [d, i32, d, i32], i32
        L.orc_quantize.argtypes, L.orc_quantize.restype = [p, i64, i64, i32, i32, f, p, p], i32
        L.orc_dequantize.argtypes, L.orc_dequantize.restype = [p, p, i64, i64, i32, d, p], None
        L.orc_swizzle_offset.argtypes, L.orc_swizzle_offset.restype = [i64, i64, i64], i64
        L.orc_swizzled_bytes.argtypes, L.orc_swizzled_bytes.restype = [i64, i64], i64
        L.orc_swizzle.argtypes, L.orc_swizzle.restype = [p, i64, i64, p], None
        L.orc_unswizzle.argtypes, L.orc_unswizzle.restype = [p, i64, i64, p], None
        L.orc_global_scale.argtypes, L.orc_global_scale.restype = [p, i64, p], f
        L.orc_gemm.argtypes = [p, p, p, p, d, d, i64, i64, i64, i32, p, i64, p, i64, p, p]
        L.orc_gemm.restype = i32
        L.orc_gemm_mt.argtypes = [p, p, p, p, d, d, i64, i64, i64, i32, p, i64, p, i64, p, p, i32]
        L.orc_gemm_mt.restype = i32
        L.orc_quantize_mt.argtypes, L.orc_quantize_mt.restype = [p, i64, i64, i32, i32, f, p, p, i32], i32
        L.orc_cpus_usable.argtypes, L.orc_cpus_usable.restype = [], i32
        L.orc_cpus_online.argtypes, L.orc_cpus_online.restype = [], i32
        L.orc_gemm_w4a16.argtypes = [p, p, p, d, i64, i64, i64, i32, p, i64, p, i64, p, p]
        L.orc_gemm_w4a16.restype = i32
        L.orc_f32_to_bf16.argtypes, L.orc_f32_to_bf16.restype = [f], ctypes.c_uint16
        L.orc_fake_quantize.argtypes, L.orc_fake_quantize.restype = [p, i64, i64, i32, i32, f, p], i32
        L.orc_quantize_running.argtypes, L.orc_quantize_running.restype = [p, i64, i64, f, p, p, p], i32
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def block_size(fmt):
    return 16 if fmt == NVFP4 else 32


def bf16_value(bits):
    return lib().orc_bf16_value(int(bits))


def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e2m1_encode(v):
    return lib().orc_e2m1_encode(float(v))


def e4m3_value(code):
    return lib().orc_e4m3_value(int(code))


def e4m3_encode(v):
    return lib().orc_e4m3_encode(float(v))


def e8m0_value(code):
    return lib().orc_e8m0_value(int(code))


def mx_exponent(amax, fmt, rule):
    """Shared block exponent e (scale 2^e) for MXFP4 (E2M1) or MXFP8 (E4M3) elements."""
    if fmt == MXFP8:
        return lib().orc_mx_exponent(float(amax), 8, 448.0, int(rule))
    return lib().orc_mx_exponent(float(amax), 2, 6.0, int(rule))


def _bits(x):
    """Accept a uint16 numpy array of bf16 bit patterns or a torch bf16 tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def cpus_usable():
    """Logical CPUs this process may run on (its affinity mask)."""
    return lib().orc_cpus_usable()


def cpus_online():
    """Online logical CPUs of the host."""
    return lib().orc_cpus_online()


def _threads(threads):
    return cpus_usable() if threads is None else max(1, int(threads))


def quantize(x, fmt, rule=EVEN, g=1.0, threads=1):
    """x: [rows, K] bf16 -> (q, sf).  q: [rows, K/2] uint8 (FP4, low nibble first) or [rows, K]
    (MXFP8); sf: [rows, K/bs] uint8 row-major scale codes.  threads: row ranges quantized in
    parallel (None = every usable CPU); the bytes do not depend on it."""
    xb = _bits(x)
    rows, K = xb.shape
    bs = block_size(fmt)
    q = np.zeros((rows, K if fmt == MXFP8 else K // 2), dtype=np.uint8)
    sf = np.zeros((rows, K // bs), dtype=np.uint8)
    rc = lib().orc_quantize_mt(_ptr(xb), rows, K, fmt, rule, float(g), _ptr(q), _ptr(sf), _threads(threads))
    if rc == -1:
        raise ValueError("K=%d is not a multiple of the block size %d" % (K, bs))
    if rc != 0:
        raise RuntimeError("oracle quantize could not start its threads")
    return q, sf


def dequantize(q, sf, K, fmt, g=1.0):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = q.shape[0]
    out = np.zeros((rows, K), dtype=np.float64)
    lib().orc_dequantize(_ptr(q), _ptr(sf), rows, K, fmt, float(g), _ptr(out))
    return out


def swizzle_offset(r, c, kblocks):
    return lib().orc_swizzle_offset(int(r), int(c), int(kblocks))


def swizzled_bytes(rows, kblocks):
    return lib().orc_swizzled_bytes(int(rows), int(kblocks))


def swizzle(sf):
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, kb = sf.shape
    out = np.zeros(swizzled_bytes(rows, kb), dtype=np.uint8)
    lib().orc_swizzle(_ptr(sf), rows, kb, _ptr(out))
    return out


def unswizzle(sw, rows, kblocks):
    sw = np.ascontiguousarray(sw, dtype=np.uint8)
    out = np.zeros((rows, kblocks), dtype=np.uint8)
    lib().orc_unswizzle(_ptr(sw), rows, kblocks, _ptr(out))
    return out


def global_scale(x):
    """NVFP4 global scale fl(amax/2688) in fp32, and the tensor amax."""
    xb = _bits(x).reshape(-1)
    amax = ctypes.c_float(0.0)
    g = lib().orc_global_scale(_ptr(xb), xb.size, ctypes.byref(amax))
    return np.float32(g), np.float32(amax.value)


def gemm(Aq, Asf, Bq, Bsf, M, N, K, fmt, gA=1.0, gB=1.0, rows=None, cols=None, threads=1):
    """fp64 reference of Out = alpha * dq(A) @ dq(B)^T on the selected rows/cols.
    Returns (out, abs_sum), both [len(rows), len(cols)] float64.  threads: output column ranges
    computed in parallel (None = every usable CPU); the values do not depend on it."""
    Aq, Asf, Bq, Bsf = (np.ascontiguousarray(a, dtype=np.uint8) for a in (Aq, Asf, Bq, Bsf))
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nr = M if r is None else r.size
    nc = N if c is None else c.size
    out = np.zeros((nr, nc), dtype=np.float64)
    absout = np.zeros((nr, nc), dtype=np.float64)
    rc = lib().orc_gemm_mt(_ptr(Aq), _ptr(Asf), _ptr(Bq), _ptr(Bsf), float(gA), float(gB), M, N, K, fmt,
                           None if r is None else _ptr(r), nr, None if c is None else _ptr(c), nc,
                           _ptr(out), _ptr(absout), _threads(threads))
    if rc != 0:
        raise MemoryError("oracle gemm allocation failed")
    return out, absout


def gemm_w4a16(A, Bq, Bsf, M, N, K, fmt, gB=1.0, rows=None, cols=None):
    """fp64 reference of Out = alpha * A @ dq(B)^T with A in bf16 (weight-only / W4A16 mode).
    Returns (out, abs_sum), both [len(rows), len(cols)] float64."""
    Ab = _bits(A)
    Bq, Bsf = (np.ascontiguousarray(a, dtype=np.uint8) for a in (Bq, Bsf))
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = None if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    nr = M if r is None else r.size
    nc = N if c is None else c.size
    out = np.zeros((nr, nc), dtype=np.float64)
    absout = np.zeros((nr, nc), dtype=np.float64)
    rc = lib().orc_gemm_w4a16(_ptr(Ab), _ptr(Bq), _ptr(Bsf), float(gB), M, N, K, fmt,
                              None if r is None else _ptr(r), nr, None if c is None else _ptr(c), nc,
                              _ptr(out), _ptr(absout))
    if rc != 0:
        raise MemoryError("oracle gemm allocation failed")
    return out, absout


def f32_to_bf16(v):
    return lib().orc_f32_to_bf16(float(v))


def fake_quantize(x, fmt, rule=EVEN, g=1.0):
    """Quantize-dequantize x [rows, K] bf16 -> bf16 bit patterns (uint16) of the same shape."""
    xb = _bits(x)
    rows, K = xb.shape
    out = np.zeros((rows, K), dtype=np.uint16)
    rc = lib().orc_fake_quantize(_ptr(xb), rows, K, fmt, rule, float(g), _ptr(out))
    if rc != 0:
        raise ValueError("K=%d is not a multiple of the block size" % K)
    return out


def quantize_running(x, amax_in):
    """NVFP4 codes/scales with g = amax_in/2688, and the updated running amax."""
    xb = _bits(x)
    rows, K = xb.shape
    q = np.zeros((rows, K // 2), dtype=np.uint8)
    sf = np.zeros((rows, K // 16), dtype=np.uint8)
    out = ctypes.c_float(0.0)
    rc = lib().orc_quantize_running(_ptr(xb), rows, K, float(amax_in), ctypes.byref(out), _ptr(q), _ptr(sf))
    if rc != 0:
        raise ValueError("K=%d is not a multiple of 16" % K)
    return q, sf, np.float32(out.value)
