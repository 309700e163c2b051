"""CPU checks of the C ABI: the library loads, exports every function include/mxq.h declares,
and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

from nvfp4_block_scaled_mx_b200 import build as mxq_build
from nvfp4_block_scaled_mx_b200 import mxq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    mxq_build.build()
    return mxq.lib()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        txt = open(os.path.join(ROOT, "include", h)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(mxq_\w+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(mxq.SIGNATURES), "binding and header disagree"


def test_size_helpers(L):
    n = ctypes.c_size_t()
    assert L.mxq_sf_bytes(8192, 5120, mxq.MXFP4, mxq.SF_SWIZZLED, ctypes.byref(n)) == 0 and n.value == 8192 * 160
    assert L.mxq_sf_bytes(130, 320, mxq.MXFP4, mxq.SF_SWIZZLED, ctypes.byref(n)) == 0 and n.value == 256 * 12
    assert L.mxq_sf_bytes(130, 320, mxq.NVFP4, mxq.SF_ROWMAJOR, ctypes.byref(n)) == 0 and n.value == 130 * 20
    assert L.mxq_q_bytes(10, 64, mxq.MXFP8, ctypes.byref(n)) == 0 and n.value == 640
    assert L.mxq_q_bytes(10, 64, mxq.NVFP4, ctypes.byref(n)) == 0 and n.value == 320
    assert L.mxq_block_size(mxq.NVFP4) == 16 and L.mxq_block_size(mxq.MXFP4) == 32
    ws = L.mxq_linear_workspace_size(8192, 5120, mxq.MXFP4)
    assert ws == 8192 * 2560 + 8192 * 160
    assert L.mxq_linear_workspace_size(0, 5120, mxq.MXFP4) == 0
    assert L.mxq_linear_kernel_count(32, 5120, 96, mxq.MXFP4) == -2  # K % 64, rejected before any device check
    assert L.mxq_linear_kernel_count(0, 5120, 5120, mxq.MXFP4) == -2
    # every dimension is bounded (1 <= v < 2^31) before any product of two is formed
    big = 1 << 40
    assert L.mxq_sf_bytes(big, big, mxq.MXFP4, mxq.SF_SWIZZLED, ctypes.byref(n)) == -2
    assert L.mxq_sf_bytes(8, 1 << 31, mxq.MXFP4, mxq.SF_ROWMAJOR, ctypes.byref(n)) == -2
    assert L.mxq_q_bytes(big, 64, mxq.MXFP4, ctypes.byref(n)) == -2
    assert L.mxq_linear_workspace_size(big, big, mxq.MXFP4) == 0
    assert L.mxq_linear_workspace_size((1 << 31) - 1, 64, mxq.MXFP4) > 0


def test_host_validation_before_launch(L):
    P = 0x10000  # never dereferenced: every case below fails validation first
    s = None
    assert L.mxq_quantize(None, 4, 64, 0, 0, None, P, P, 0, s) == -1
    assert L.mxq_quantize(P, 4, 48, 0, 0, None, P, P, 0, s) == -2  # K % 32
    assert L.mxq_quantize(P, 0, 64, 0, 0, None, P, P, 0, s) == -2
    assert L.mxq_quantize(P, 1 << 40, 1 << 40, 0, 0, None, P, P, 0, s) == -2  # no int64 overflow in M * K
    assert L.mxq_quantize(P, 1 << 28, 1 << 10, 0, 0, None, P, P, 0, s) == -2  # M * K / 8 >= 2^31
    assert L.mxq_quantize(P + 8, 4, 64, 0, 0, None, P, P, 0, s) == -3
    assert L.mxq_quantize(P, 4, 64, 7, 0, None, P, P, 0, s) == -4
    assert L.mxq_quantize(P, 4, 64, 1, 0, None, P, P, 0, s) == -1  # NVFP4 needs g
    assert L.mxq_gemm(P, P, P, P, None, None, 4, 4, 96, 0, 0, P, s) == -2  # K % 64
    assert L.mxq_gemm(P, P, P, P, None, None, 4, 0, 128, 0, 0, P, s) == -2
    assert L.mxq_gemm(P, P, P, P, None, None, 4, 4, 128, 1, 0, P, s) == -1
    assert L.mxq_gemm(P, P, P + 4, P, None, None, 4, 4, 128, 0, 0, P, s) == -3
    assert L.mxq_gemm(P, P, P, P, None, None, 4, 4, 128, 0, 5, P, s) == -4
    assert L.mxq_linear(P, P, P, None, None, 4, 4, 128, 0, 1, 0, P, 16, P, s) == -5
    assert L.mxq_swizzle_scales(None, 4, 4, P, s) == -1
    assert L.mxq_global_scale(P, 0, P, P, s) == -2
    assert L.mxq_selftest_timeout(0, s) == -2
    assert L.mxq_amax(None, 4, P, s) == -1
    assert L.mxq_amax(P, 0, P, s) == -2
    assert L.mxq_amax(P + 8, 4, P, s) == -3
    # the allocation-free linear call reports mxq_linear's codes in mxq_linear's order
    assert L.mxq_linear_noalloc(P, P, P, None, None, 4, 4, 128, 7, 1, 0, P, s) == -4
    assert L.mxq_linear_noalloc(None, P, P, None, None, 4, 4, 128, 0, 1, 0, P, s) == -1
    assert L.mxq_linear_noalloc(P, P, P, None, None, 4, 4, 96, 0, 1, 0, P, s) == -2
    assert L.mxq_linear_noalloc(P, P, P, None, None, 8192, 4, 5120, 0, 1, 0, P, s) == -5
    assert L.mxq_linear(P, P, P, None, None, 4, 4, 128, 7, 1, 0, P, 1 << 20, P, s) == -4
    assert L.mxq_strerror(-5) == b"workspace too small"


# the calls of the method's hot path: each declaration's comment names the page (a quoted title)
# that defines the operation, or says that the pages do not describe it
CITED = ["mxq_quantize", "mxq_quantize_running", "mxq_fake_quantize", "mxq_swizzle_scales", "mxq_global_scale",
         "mxq_amax", "mxq_gemm", "mxq_gemm_w4a16", "mxq_linear"]


def test_header_cites_the_defining_passage():
    txt = open(os.path.join(ROOT, "include", "mxq.h")).read()
    for name in CITED:
        m = re.search(r"/\*((?:(?!\*/).)*)\*/\s*(?:#define[^\n]*\n\s*)?int %s\(" % name, txt, flags=re.S)
        assert m, "no comment block directly above %s" % name
        comment = m.group(1)
        assert re.search(r'"(Qwen3\.5|intel-ai)[^"]*"', comment.replace("\n *", " ")), "%s cites no page" % name
