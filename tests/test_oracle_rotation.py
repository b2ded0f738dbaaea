"""Pins of the oracle's block Hadamard rotation: Sylvester matrix from scipy,
orthogonality, exact products on integer inputs, a hand-worked stage-order example,
and rotation invariance of the product (XH)(WH)^T = XW^T."""
import json
import os
import struct

import numpy as np
import pytest
import scipy.linalg
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f(hexs):
    return np.array([struct.unpack(">f", bytes.fromhex(h))[0] for h in hexs], np.float32)


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32])
def test_fwht_columns_are_scaled_sylvester_hadamard(orc, n):
    H = scipy.linalg.hadamard(n).astype(np.float64)  # library Sylvester construction
    c = orc.hadamard_scale(n)
    cols = np.stack([orc.fwht(np.eye(n, dtype=np.float32)[j]) for j in range(n)], axis=1)
    assert np.array_equal(cols.astype(np.float64), (H * np.float64(np.float32(c))))
    Ho = cols.astype(np.float64) / np.float64(np.float32(c))
    assert np.array_equal(Ho @ Ho.T, n * np.eye(n))


@pytest.mark.parametrize("n", [16, 32])
def test_fwht_integer_inputs_exact(orc, n):
    rng = np.random.default_rng(n)
    H = scipy.linalg.hadamard(n).astype(np.int64)
    c = np.float32(orc.hadamard_scale(n))
    for _ in range(50):
        v = rng.integers(-1000, 1000, n)
        want = (H @ v).astype(np.float32) * c  # exact integer sum, one fp32 rounding
        got = orc.fwht(v.astype(np.float32))
        assert np.array_equal(got, want)


def test_fwht_stage_order_golden(orc):
    g = json.load(open(os.path.join(GOLDEN, "fwht_stage_order_n4.json")))
    got = orc.fwht(_f(g["input_f32_hex"]))
    assert np.array_equal(got.view(np.uint32), _f(g["expected_f32_hex"]).view(np.uint32))


@pytest.mark.parametrize("hn", [16, 32])
def test_rotate_matches_dense_blockdiag_product(orc, hn):
    x = (torch.randn(64, 128, generator=torch.Generator().manual_seed(hn)) * 3).to(torch.bfloat16)
    xf = x.float().numpy().astype(np.float64)
    H = scipy.linalg.hadamard(hn) / np.sqrt(hn)
    want_row = (xf.reshape(64, -1, hn) @ H.T).reshape(64, 128)
    got_row = orc.rotate(x, hn, orc.ROW)
    assert np.allclose(got_row, want_row, rtol=1e-5, atol=1e-5)
    want_col = (xf.T.reshape(128, -1, hn) @ H.T).reshape(128, 64)
    got_col = orc.rotate(x, hn, orc.COL)
    assert got_col.shape == (128, 64)
    assert np.allclose(got_col, want_col, rtol=1e-5, atol=1e-5)
    assert np.array_equal(orc.rotate(x, 0, orc.COL), x.float().numpy().T)


@pytest.mark.parametrize("hn", [16, 32])
def test_rotation_leaves_the_product_invariant(orc, hn):
    g = torch.Generator().manual_seed(7)
    X = torch.randn(96, 256, generator=g).to(torch.bfloat16)
    W = torch.randn(64, 256, generator=g).to(torch.bfloat16)
    ref = X.double().numpy() @ W.double().numpy().T
    rot = orc.rotate(X, hn).astype(np.float64) @ orc.rotate(W, hn).astype(np.float64).T
    err = np.linalg.norm(rot - ref) / np.linalg.norm(ref)
    assert err < 1e-6
