"""Pins of the oracle's quantiser variants: the Philox4x32-10 generator, stochastic
E2M1 rounding, randomised Hadamard signs and a caller-supplied NVFP4 tensor amax.

The pages (gist.science summary of arXiv 2605.09825, Methodology item 3 and Findings
section 2) name stochastic rounding and randomised Hadamard rotations only as the
stabilisers they reject; each check below pins the reading the oracle takes of them
against something other than the oracle itself: the generator's published
known-answer vectors, exact rational arithmetic, unbiasedness, and equivalences with
the plain (already pinned) quantiser on sign-flipped inputs."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from fp4_block_scaled_deterministic_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
MAGS = [Fraction(v) for v in ("0", "0.5", "1", "1.5", "2", "3", "4", "6")]


def test_philox_known_answers(orc):
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    for v in kat["vectors"]:
        ctr = [int(h, 16) for h in v["counter"]]
        key = [int(h, 16) for h in v["key"]]
        out = orc.philox4x32_10(ctr, key)
        assert [f"{w:08x}" for w in out] == v["output"]


def test_philox_words_are_uniform(orc):
    """Words drawn over consecutive indices of one stream look uniform: mean of the
    top-24-bit fraction and the rate of bit 31 (the sign draw) within 5 sigma."""
    n = 20000
    w = np.array([orc.philox_word(12345, i, 0) for i in range(n)], np.uint64)
    u = (w >> 8).astype(np.float64) / 2.0**24
    assert abs(u.mean() - 0.5) < 5 * np.sqrt(1 / 12 / n)
    assert abs((w >> 31).mean() - 0.5) < 5 * 0.5 / np.sqrt(n)
    # streams and seeds give different words for the same index
    assert orc.philox_word(1, 7, 0) != orc.philox_word(1, 7, 1)
    assert orc.philox_word(1, 7, 0) != orc.philox_word(2, 7, 0)


def _sr_exact(q: float, w: int) -> int:
    """Stochastic rounding decided in exact rational arithmetic."""
    a = abs(Fraction(q))
    sign = 8 if np.signbit(np.float32(q)) else 0
    if a >= 6:
        return sign | 7
    lo = max(i for i, m in enumerate(MAGS) if m <= a)
    p = (a - MAGS[lo]) / (MAGS[lo + 1] - MAGS[lo])
    return sign | (lo + 1 if Fraction(w >> 8, 2**24) < p else lo)


def test_stochastic_rounding_matches_exact_rational_rule(orc):
    rng = np.random.default_rng(3)
    qs = list(rng.uniform(-7, 7, 3000).astype(np.float32))
    qs += [np.float32(k / 64) for k in range(-450, 451)]  # grid points and fine fractions
    qs += [np.float32(m) * s for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) for s in (1, -1)]
    for q in qs:
        for w in (0, 0xFFFFFFFF, int(rng.integers(0, 2**32)), int(rng.integers(0, 2**32))):
            assert orc.e2m1_encode_sr(float(q), w) == _sr_exact(float(q), w), (q, w)


def test_stochastic_rounding_keeps_representable_values(orc):
    for m in range(8):
        v = float(MAGS[m])
        for w in (0, 1 << 8, 0x80000000, 0xFFFFFFFF):
            assert orc.e2m1_encode_sr(v, w) == m
            assert orc.e2m1_encode_sr(-v, w) == 8 | m
    assert orc.e2m1_encode_sr(6.5, 0) == 7 and orc.e2m1_encode_sr(-100.0, 0) == 15


def test_stochastic_rounding_is_unbiased(orc):
    """Over all 2^24 fractions u (every 4097th one here), the mean of the rounded value
    equals q up to the 2^-24 granularity of u."""
    for q in (0.3, 0.9, 1.3, 2.2, 3.7, 4.9, 5.99):
        ks = np.arange(0, 2**24, 4097, dtype=np.int64)
        vals = [orc.e2m1_decode(orc.e2m1_encode_sr(q, int(k) << 8)) for k in ks]
        assert abs(np.mean(vals) - np.float32(q)) < 2 * 2.0 / len(ks) ** 0.5 * 0.5 + 1e-3


def _x(rows, cols, seed):
    return synthetic.normal(rows, cols, 1.0, seed=seed, outlier_frac=0.01, outlier_mult=30.0)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("axis", [0, 1])
def test_quantize_sr_rounds_each_code_to_a_neighbour(orc, fmt, axis):
    """SR changes no block scale, and each code is one of the two E2M1 neighbours of
    its quotient (so it differs from the nearest code by at most one step)."""
    x = _x(64, 128, 1)
    cn, sn, Sn, An = orc.quantize(x, fmt, 16, axis)
    cs, ss, Ss, As = orc.quantize(x, fmt, 16, axis, sr_seed=99)
    assert np.array_equal(sn, ss) and Sn == Ss and An == As
    dn = orc.dequantize(cn, sn, Sn, fmt)
    ds = orc.dequantize(cs, ss, Ss, fmt)
    # neighbouring E2M1 values are at most 2 apart in units of the block scale
    R, C = dn.shape
    bs = orc.BLOCK[fmt]
    for r in range(R):
        for kb in range(C // bs):
            sb = int(sn[orc.scale_offset(r, kb, C // bs)])
            unit = 2.0 ** (sb - 127) if fmt == 0 else orc.e4m3_decode(sb) * Sn
            sl = slice(kb * bs, (kb + 1) * bs)
            assert np.all(np.abs(dn[r, sl] - ds[r, sl]) <= 2 * unit)
    assert not np.array_equal(cn, cs)


def test_quantize_sr_draw_index_and_determinism(orc):
    """Element (i, c) of the quantised matrix draws word(seed, i*C + c, 1 + axis):
    recomputed here from the quotient of the (pinned) nearest-rounding path."""
    x = _x(32, 64, 2)
    for axis in (0, 1):
        cs, ss, _, _ = orc.quantize(x, 0, 0, axis, sr_seed=7)
        assert np.array_equal(cs, orc.quantize(x, 0, 0, axis, sr_seed=7)[0])
        assert not np.array_equal(cs, orc.quantize(x, 0, 0, axis, sr_seed=8)[0])
        v = orc.rotate(x, 0, axis)
        R, C = v.shape
        for (i, c) in ((0, 0), (3, 17), (R - 1, C - 1), (5, C - 31)):
            blk = v[i, c // 32 * 32:c // 32 * 32 + 32]
            e = int(orc.mx_scale_exponent(np.float32(np.max(np.abs(blk)))).item())
            q = np.float32(v[i, c] * np.float32(2.0**-e))
            w = orc.philox_word(7, i * C + c, 1 + axis)
            nib = (cs[i, c // 2] >> (4 * (c & 1))) & 15
            assert nib == orc.e2m1_encode_sr(float(q), w)


def test_quantize_sr_is_unbiased_over_seeds(orc):
    """Averaged over seeds, the dequantised SR tensor approaches the rotated tensor,
    while nearest rounding keeps a fixed error."""
    x = _x(32, 64, 3)
    v = orc.rotate(x, 16, 0).astype(np.float64)
    acc = np.zeros_like(v)
    n = 64
    for seed in range(n):
        c, s, _, _ = orc.quantize(x, 0, 16, 0, sr_seed=seed)
        acc += orc.dequantize(c, s, None, 0)
    c, s, _, _ = orc.quantize(x, 0, 16, 0)
    # compare where no clipping happens (|v| < 6 * block scale): clipping biases both
    R, C = v.shape
    scale = np.array([[2.0 ** (int(s[orc.scale_offset(r, k // 32, C // 32)]) - 127)
                       for k in range(C)] for r in range(R)])
    keep = np.abs(v) < 6 * scale
    assert keep.mean() > 0.9
    err_rne = np.linalg.norm((orc.dequantize(c, s, None, 0) - v)[keep])
    err_mean = np.linalg.norm((acc / n - v)[keep])
    # nearest rounding: rms ~ step/sqrt(12); the SR mean: rms ~ step*sqrt(1/6/n)
    assert err_mean < 0.35 * err_rne


def _flip_bf16(x: torch.Tensor, neg: np.ndarray, axis: int) -> torch.Tensor:
    """x with the columns (axis ROW) or rows (axis COL) marked in neg negated; exact."""
    bits = x.view(torch.int16).numpy().view(np.uint16).copy()
    if axis == 0:
        bits[:, neg] ^= 0x8000
    else:
        bits[neg, :] ^= 0x8000
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hn", [16, 32])
def test_rht_equals_plain_rotation_of_sign_flipped_input(orc, fmt, axis, hn):
    """Randomised Hadamard = the plain quantiser applied to x with every element at
    contraction index j negated when bit 31 of word(seed, j, 0) is set."""
    x = _x(64, 96, 4)
    n_axis = x.shape[1] if axis == 0 else x.shape[0]
    neg = np.array([orc.philox_word(21, j, 0) >> 31 for j in range(n_axis)], bool)
    assert 0.3 < neg.mean() < 0.7
    got = orc.quantize(x, fmt, hn, axis, rht_seed=21)
    ref = orc.quantize(_flip_bf16(x, neg, axis), fmt, hn, axis)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    assert got[2] == ref[2] and got[3] == ref[3]
    assert orc.rotated_amax(x, hn, axis, rht_seed=21) == orc.rotated_amax(_flip_bf16(x, neg, axis), hn, axis)


def test_rht_rotation_is_the_block_matrix_product(orc):
    """Small-integer inputs (exact in fp32): rotate with signs = x diag(s) H_blk c in fp64."""
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-8, 9, (8, 64), generator=g).to(torch.bfloat16)
    for hn in (16, 32):
        s = np.array([-1.0 if orc.rht_negate(77, j) else 1.0 for j in range(64)])
        blk = scipy.linalg.block_diag(*([scipy.linalg.hadamard(hn)] * (64 // hn)))
        sums = (x.float().numpy().astype(np.float64) * s) @ blk.T   # exact small integers
        ref = sums.astype(np.float32) * np.float32(orc.hadamard_scale(hn))  # one fp32 rounding
        assert np.array_equal(orc.rotate(x, hn, 0, rht_seed=77), ref)


def test_rht_preserves_the_product():
    """(X D H)(W D H)^T = X W^T: both operands of a pass share the seed."""
    from oracle import rotate
    X = _x(32, 128, 6)
    W = synthetic.normal(48, 128, 0.02, seed=7)
    ref = X.double().numpy() @ W.double().numpy().T
    for hn in (16, 32):
        got = rotate(X, hn, 0, rht_seed=3).astype(np.float64) @ rotate(W, hn, 0, rht_seed=3).astype(np.float64).T
        assert np.max(np.abs(got - ref)) < 1e-5 * np.max(np.abs(ref))
        bad = rotate(X, hn, 0, rht_seed=3).astype(np.float64) @ rotate(W, hn, 0, rht_seed=4).astype(np.float64).T
        assert np.max(np.abs(bad - ref)) > 1e-2 * np.max(np.abs(ref))


def test_supplied_amax_equals_computed_and_scales_with_it(orc):
    x = _x(64, 64, 8)
    for axis in (0, 1):
        c, s, S, T = orc.quantize(x, 1, 16, axis)
        c2, s2, S2, T2 = orc.quantize(x, 1, 16, axis, amax=T)
        assert np.array_equal(c, c2) and np.array_equal(s, s2) and S == S2 and T2 == T
        # a larger supplied amax gives the tensor scale T'/2688 and a valid quantisation
        c3, s3, S3, T3 = orc.quantize(x, 1, 16, axis, amax=4 * T)
        assert T3 == np.float32(4 * T) and S3 == np.float32(np.float32(4 * T) / np.float32(2688))
