"""Scalar CPU oracle for the microscaling W4A4 linear layer (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package.  The product library never loads it.  The arithmetic lives in ``mxq_oracle.c``;
this module builds it with gcc and wraps it with ctypes over numpy arrays.
"""
from .oracle import (  # noqa: F401
    MXFP4, NVFP4, MXFP8, EVEN, CEIL, build, lib, block_size,
    bf16_value, e2m1_value, e2m1_encode, e4m3_value, e4m3_encode, e8m0_value, mx_exponent,
    quantize, dequantize, swizzle, unswizzle, swizzle_offset, swizzled_bytes, global_scale, gemm, gemm_w4a16,
    f32_to_bf16, fake_quantize, quantize_running, cpus_usable, cpus_online,
)
