"""The oracle's threaded quantizer and GEMM give exactly the single-threaded results: each thread
runs the single-threaded code on its own range of rows (quantizer) or output columns (GEMM), so no
byte or value may depend on the thread count.  Row and column selections, ragged splits (more
threads than rows or columns) and every format are covered."""
import numpy as np
import pytest

import oracle
from nvfp4_block_scaled_mx_b200 import synth


@pytest.mark.parametrize("fmt,rule", [(oracle.MXFP4, oracle.CEIL), (oracle.NVFP4, oracle.EVEN),
                                      (oracle.MXFP8, oracle.EVEN)])
def test_thread_count_does_not_change_results(fmt, rule):
    M, N, K = 37, 70, 320
    A = synth.random_bf16((M, K), 41)
    W = synth.random_bf16((N, K), 42, std=0.02)
    g = 1.0
    if fmt == oracle.NVFP4:
        g = float(oracle.global_scale(A)[0])
    base = None
    for t in (1, 2, 3, 8, 100):
        qa, sa = oracle.quantize(A, fmt, rule, g=g, threads=t)
        qw, sw = oracle.quantize(W, fmt, oracle.EVEN, g=g, threads=t)
        rows = np.array([0, 5, 36], dtype=np.int64)
        cols = np.array([1, 2, 69, 33], dtype=np.int64)
        full, full_abs = oracle.gemm(qa, sa, qw, sw, M, N, K, fmt, gA=g, gB=g, threads=t)
        sel, sel_abs = oracle.gemm(qa, sa, qw, sw, M, N, K, fmt, gA=g, gB=g, rows=rows, cols=cols, threads=t)
        assert np.array_equal(sel, full[np.ix_(rows, cols)]) and np.array_equal(sel_abs, full_abs[np.ix_(rows, cols)])
        got = (qa, sa, qw, sw, full, full_abs)
        if base is None:
            base = got
        else:
            for x, y in zip(base, got):
                assert np.array_equal(x, y)


def test_transposed_product_is_the_same_sum():
    """out^T = dq(B) dq(A)^T term by term: the full-size parity tests take all rows of a few columns
    from the oracle run with the operands swapped."""
    M, N, K = 9, 13, 256
    qa, sa = oracle.quantize(synth.random_bf16((M, K), 43), oracle.MXFP4, oracle.CEIL)
    qw, sw = oracle.quantize(synth.random_bf16((N, K), 44, std=0.02), oracle.MXFP4, oracle.EVEN)
    out, ab = oracle.gemm(qa, sa, qw, sw, M, N, K, oracle.MXFP4)
    out_t, ab_t = oracle.gemm(qw, sw, qa, sa, N, M, K, oracle.MXFP4, threads=4)
    assert np.array_equal(out, out_t.T) and np.array_equal(ab, ab_t.T)


def test_cpu_counts():
    assert 1 <= oracle.cpus_usable() <= oracle.cpus_online()
