"""Pins of the oracle's MXFP8 comparator quantiser (E4M3 elements under an E8M0 scale
per 32 elements; reading R15 in the oracle header): the scale exponent invariant, the
element codes against a library E4M3 conversion, exact round trips of representable
blocks, and the GEMM entries against dequantise-then-multiply."""
import ml_dtypes
import numpy as np
import pytest
import torch

from fp4_block_scaled_deterministic_b200 import synthetic

MXFP8 = 2


def _x(rows, cols, seed, mult=30.0):
    return synthetic.normal(rows, cols, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=mult)


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hn", [0, 16, 32])
def test_mxfp8_scale_and_codes(orc, axis, hn):
    x = _x(96, 160, seed=3 + hn)
    codes, scales, _, _ = orc.quantize(x, MXFP8, hn, axis)
    v = orc.rotate(x, hn, axis)
    R, C = v.shape
    assert codes.shape == (R, C)
    for r in range(R):
        for kb in range(C // 32):
            blk = v[r, 32 * kb:32 * kb + 32]
            amax = float(np.max(np.abs(blk)))
            e = int(scales[orc.scale_offset(r, kb, C // 32)]) - 127
            if amax == 0:
                assert e == -127
                continue
            assert 256 <= amax * 2.0 ** -e < 512          # floor(log2 amax) - 8
            q = np.clip(blk.astype(np.float32) * np.float32(2.0 ** -e), -448, 448)
            ref = q.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            assert np.array_equal(codes[r, 32 * kb:32 * kb + 32], ref)


def test_mxfp8_round_trip_of_representable_blocks(orc):
    rng = np.random.default_rng(4)
    e4m3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    finite = e4m3[np.isfinite(e4m3)]
    rows = []
    for k in range(-20, 20, 3):
        c = rng.choice(finite, 32)
        c[rng.integers(0, 32)] = rng.choice([256.0, 288.0, 320.0, 448.0, -448.0])
        rows.append(c * 2.0 ** k)
    x = torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)
    # every value above has at most 4 significant bits, so the bf16 cast is exact
    assert np.array_equal(x.float().numpy().astype(np.float64), np.array(rows))
    codes, scales, _, _ = orc.quantize(x, MXFP8, 0, 0)
    assert np.array_equal(orc.dequantize(codes, scales, None, MXFP8), np.array(rows))


def test_mxfp8_gemm_entries_match_dequantised_product(orc):
    X = _x(64, 96, seed=5)
    W = synthetic.normal(48, 96, 0.02, seed=6)
    a = orc.quantize(X, MXFP8, 16, 0)[:3]
    b = orc.quantize(W, MXFP8, 16, 0)[:3]
    full = orc.dequantize(*a, MXFP8) @ orc.dequantize(*b, MXFP8).T
    ms = np.array([0, 5, 63, 17]), np.array([0, 47, 3, 20])
    got = orc.gemm_entries(a, b, MXFP8, *ms)
    assert np.allclose(got, full[ms[0], ms[1]], rtol=1e-12, atol=0)
    # MXFP8 is far closer to the unquantised product than MXFP4
    exact = X.double().numpy() @ W.double().numpy().T
    q4 = orc.dequantize(*orc.quantize(X, 0, 16, 0)[:3], 0) @ orc.dequantize(*orc.quantize(W, 0, 16, 0)[:3], 0).T
    err8 = np.linalg.norm(full - exact) / np.linalg.norm(exact)
    err4 = np.linalg.norm(q4 - exact) / np.linalg.norm(exact)
    assert err8 < 0.5 * err4
