"""B200 (sm_100a) microscaling W4A4 linear layer: MXFP4 / NVFP4 / MXFP8 quantizer, scale swizzle,
tcgen05 block-scaled GEMM and the fused quantize-then-GEMM linear, behind the C ABI of libmxq.so."""
from . import mxq  # noqa: F401
