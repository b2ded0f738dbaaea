"""Pins of the oracle's GEMM: exact on integer-valued operands against numpy's
integer matmul, equal to numpy's fp64 matmul on random ones, and the entry-wise
evaluation from quantised operands equal to dequantise-then-multiply."""
import numpy as np
import pytest

from fp4_block_scaled_deterministic_b200 import synthetic


def test_gemm_integer_exact(orc):
    rng = np.random.default_rng(8)
    A = rng.integers(-6, 7, (40, 96))
    B = rng.integers(-6, 7, (24, 96))
    C = orc.gemm_f64(A.astype(np.float64), B.astype(np.float64))
    assert np.array_equal(C, (A @ B.T).astype(np.float64))


def test_gemm_matches_library_fp64(orc):
    rng = np.random.default_rng(9)
    A = rng.standard_normal((33, 70))
    B = rng.standard_normal((17, 70))
    C = orc.gemm_f64(A, B)
    assert np.allclose(C, A @ B.T, rtol=1e-13, atol=1e-13)
    assert orc.gemm_f64(A, B).shape == (33, 17)


@pytest.mark.parametrize("fmt,hn", [(0, 16), (1, 16), (0, 32), (1, 0)])
def test_gemm_entries_equal_dequantised_product(orc, fmt, hn):
    X = synthetic.normal(64, 256, 1.0, seed=1, outlier_frac=0.01, outlier_mult=30)
    W = synthetic.normal(96, 256, 0.02, seed=2)
    xq = orc.quantize(X, fmt, hn)[:3]
    wq = orc.quantize(W, fmt, hn)[:3]
    full = orc.gemm_f64(orc.dequantize(*xq, fmt), orc.dequantize(*wq, fmt))
    rng = np.random.default_rng(10)
    ms, ns = rng.integers(0, 64, 200), rng.integers(0, 96, 200)
    ent = orc.gemm_entries(xq, wq, fmt, ms, ns)
    assert np.allclose(ent, full[ms, ns], rtol=1e-12, atol=1e-12)


def test_quantised_gemm_tracks_unquantised(orc):
    """Information-level sanity: the FP4 product is close to the bf16 product."""
    X, W = synthetic.tiny_linear()
    ref = X.double().numpy() @ W.double().numpy().T
    xq = orc.quantize(X, orc.MXFP4, 16)[:3]
    wq = orc.quantize(W, orc.MXFP4, 16)[:3]
    C = orc.gemm_f64(orc.dequantize(*xq, orc.MXFP4), orc.dequantize(*wq, orc.MXFP4))
    rel = np.linalg.norm(C - ref) / np.linalg.norm(ref)
    assert rel < 0.2
