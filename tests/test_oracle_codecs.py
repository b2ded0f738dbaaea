"""Pins of the oracle's element and scale codecs against things other than itself:
library routines (ml_dtypes), exhaustive nearest-value search, closed forms and
invariants of the formats."""
import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _lib_e2m1(q):
    return np.asarray(q, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


# ------------------------------------------------------------------ E2M1

def test_e2m1_table_matches_library(orc):
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    mine = np.array([orc.e2m1_decode(int(c)) for c in codes])
    assert np.array_equal(np.signbit(lib), np.signbit(mine))
    assert np.array_equal(lib, mine)
    assert sorted(set(np.abs(mine))) == E2M1_VALUES


def _nearest_even(q):
    """Brute force: nearest of the 8 magnitudes, ties to the even index, sign kept."""
    a = abs(float(q))
    best = min(range(8), key=lambda i: (abs(a - E2M1_VALUES[i]), i % 2))
    return (8 if math.copysign(1.0, float(q)) < 0 else 0) | best


def test_e2m1_rne_grid_bruteforce(orc):
    q = np.array([k / 64 for k in range(-512, 513)], np.float32)
    mine = orc.e2m1_encode(q)
    assert np.array_equal(mine, _lib_e2m1(q))
    assert all(int(m) == _nearest_even(v) for m, v in zip(mine, q))


def test_e2m1_midpoints_and_neighbours(orc):
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = []
    for m in mids:
        m = np.float32(m)
        vals += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(10))]
    vals = np.array(vals + [-v for v in vals], np.float32)
    mine = orc.e2m1_encode(vals)
    assert np.array_equal(mine, _lib_e2m1(vals))
    # ties go to the even magnitude index
    assert [int(c) for c in orc.e2m1_encode(np.array(mids, np.float32))] == [0, 2, 2, 4, 4, 6, 6]


def test_e2m1_saturation_signed_zero_random(orc):
    rng = np.random.default_rng(0)
    special = np.array([0.0, -0.0, 1e-40, -1e-40, 6.0, 6.5, 7.0, 8.0, 1e30, -1e30, 3.4e38],
                       np.float32)
    rand = (rng.standard_normal(20000) * np.exp2(rng.integers(-8, 8, 20000))).astype(np.float32)
    q = np.concatenate([special, rand])
    mine = orc.e2m1_encode(q)
    assert np.array_equal(mine, _lib_e2m1(q))
    assert int(orc.e2m1_encode(np.array([-0.0], np.float32))[0]) == 8   # sign kept
    assert int(orc.e2m1_encode(np.array([1e30], np.float32))[0]) == 7    # satfinite


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_all_codes_match_library(orc):
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mine = np.array([orc.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(mine))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(lib[~nan], mine[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x38] == 1.0


def test_e4m3_encode_roundtrip_every_code(orc):
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = np.float32(orc.e4m3_decode(c))
        if c == 0x80:  # -0 keeps its sign
            assert int(orc.e4m3_encode([-0.0])[0]) == 0x80
            continue
        assert int(orc.e4m3_encode([v])[0]) == c, hex(c)


def test_e4m3_midpoints_ties_to_even(orc):
    vals = [orc.e4m3_decode(c) for c in range(0x7F)]
    for lo in range(0x7E):
        mid = (vals[lo] + vals[lo + 1]) / 2  # exact in fp32 (<= 5 significant bits)
        got = int(orc.e4m3_encode([mid])[0])
        assert got == (lo if lo % 2 == 0 else lo + 1), (lo, mid, got)


def test_e4m3_encode_matches_library_and_saturates(orc):
    rng = np.random.default_rng(1)
    t = np.abs(rng.standard_normal(50000) * np.exp2(rng.integers(-14, 9, 50000))).astype(np.float32)
    t = t[t <= 464.0]  # the library rounds >464 to NaN; the oracle saturates
    mine = orc.e4m3_encode(t)
    lib = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(mine, lib)
    big = np.array([448.0, 449.0, 464.0, 465.0, 1e9, np.inf], np.float32)
    assert list(orc.e4m3_encode(big)) == [0x7E] * 6
    assert int(orc.e4m3_encode([np.nan])[0]) == 0x7F


# ------------------------------------------------------------------ E8M0

def test_mx_exponent_invariant(orc):
    rng = np.random.default_rng(2)
    a = (rng.uniform(1.0, 2.0, 40000) * np.exp2(rng.integers(-125, 127, 40000))).astype(np.float32)
    e = orc.mx_scale_exponent(a)
    scaled = a.astype(np.float64) * np.exp2(-e.astype(np.float64))
    assert np.all((scaled >= 4.0) & (scaled < 8.0))


def test_mx_exponent_edges(orc):
    f32 = np.float32
    cases = {0.0: -127, 1e-45: -127, 1e-39: -127, float(f32(2.0 ** -125)): -127,
             float(f32(2.0 ** -124)): -126, 6.0: 0, 4.0: 0, float(np.nextafter(f32(4), f32(0))): -1,
             float(np.finfo(np.float32).max): 125}
    for a, e in cases.items():
        assert int(orc.mx_scale_exponent([a])[0]) == e, (a, e)


# ------------------------------------------------------------------ rotation constant

def test_hadamard_constants_are_correctly_rounded(orc):
    assert orc.hadamard_scale(16) == 0.25
    c32 = orc.hadamard_scale(32)
    # |c32 - 1/sqrt(32)| <= half an ulp, checked with exact rationals:
    # (c32 - d)^2 vs 1/32 bracketing: c32 is RN iff 1/32 lies between (c32 -+ ulp/2)^2
    ulp = Fraction(np.spacing(np.float32(c32)).item())
    c = Fraction(float(np.float32(c32)))
    lo, hi = c - ulp / 2, c + ulp / 2
    assert lo * lo < Fraction(1, 32) < hi * hi
