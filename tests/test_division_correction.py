"""The NVFP4 quantiser forms each quotient RN(v/d) from y = RN(1/d) by two correction
steps: q0 = RN(v*y); q1 = RN(q0 + RN(v - q0*d)*y), which is faithful; then the step of
Markstein (IBM J. Res. Dev. 34(1), 1990) with the exact residual r = v - q1*d:
q = RN(q1 + r*y). One step from q0 is not enough: q0 can be just over one ulp from v/d
(this test found such a case).

Checked here in exact rational arithmetic, with fp32 round-to-nearest-even written out:
the residual is representable and q is the correctly rounded quotient, over the
kernel's operating range: d = RN(E4M3 value * S) with 2^-100 <= d <= 2^100 and
quotients up to ~8: random, at the bottom of each binade (where v*y errs most) and
within a few ulps of every E2M1 rounding threshold. (The kernels' own outputs are
compared with the oracle's IEEE divisions in the GPU parity tests.)"""
from fractions import Fraction

import numpy as np

THRESHOLDS = [Fraction(1, 4), Fraction(3, 4), Fraction(5, 4), Fraction(7, 4),
              Fraction(5, 2), Fraction(7, 2), Fraction(5)]


def rn32(x: Fraction) -> Fraction:
    """x rounded to the nearest fp32 value, ties to even (no overflow in this range)."""
    if x == 0:
        return Fraction(0)
    s = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** (max(e, -126) - 23)
    m = a / ulp
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return s * n * ulp


def exact(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def corrected_quotient(v: Fraction, d: Fraction):
    y = rn32(1 / d)
    q0 = rn32(v * y)                 # can be just over one ulp from v/d
    q1 = rn32(q0 + rn32(v - q0 * d) * y)  # within about half an ulp: faithful
    r = v - q1 * d
    assert rn32(r) == r, "residual not representable"
    return rn32(q1 + r * y)


def fma_sequence(v: Fraction, d: Fraction) -> Fraction:
    """The kernel's instructions as written, one rounding per FMA (no exactness assumed)."""
    y = rn32(1 / d)
    q0 = rn32(v * y)
    q1 = rn32(q0 + rn32(v - q0 * d) * y)
    return rn32(q1 + rn32(v - q1 * d) * y)


def e4m3_values():
    vals = []
    for e in range(-6, 9):
        for m in range(8):
            vals.append(Fraction(8 + m, 8) * Fraction(2) ** e)
    vals += [Fraction(m, 8) * Fraction(2) ** -6 for m in range(1, 8)]  # subnormals
    return [v for v in vals if v <= 448]


def test_correction_step_is_correctly_rounded():
    rng = np.random.default_rng(7)
    scales = e4m3_values()
    checked = 0
    for _ in range(400):
        S = exact(np.float32(2.0) ** rng.uniform(-60, 60) * rng.uniform(1, 2))
        d = rn32(scales[rng.integers(len(scales))] * S)
        if not (Fraction(2) ** -100 <= d <= Fraction(2) ** 100):
            continue
        cases = []
        for _ in range(20):  # random quotients in [0, 8)
            cases.append(rn32(Fraction(float(rng.uniform(-8, 8))) * d))
        for e in range(-3, 3):  # the bottom 3% of each binade 2^-3 .. 2^3
            for _ in range(4):
                cases.append(rn32(Fraction(float(rng.uniform(1, 1.03))) * Fraction(2) ** e * d))
        for t in THRESHOLDS:  # quotients within a few ulps of each threshold
            base = rn32(t * d)
            ulp = Fraction(2) ** ((base.numerator.bit_length() - base.denominator.bit_length()) - 24)
            for k in range(-6, 7):
                for sgn in (1, -1):
                    cases.append(sgn * rn32(base + k * ulp))
        for v in cases:
            assert corrected_quotient(v, d) == rn32(v / d), (v, d)
            checked += 1
    assert checked > 30000


E2M1_GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2),
             Fraction(3), Fraction(4), Fraction(6)]


def e2m1_magnitude_code(m: Fraction) -> int:
    """Index of the E2M1 magnitude that m >= 0 rounds to (nearest, ties to the even
    code, saturating at 6)."""
    for k in range(7):
        lo, hi = E2M1_GRID[k], E2M1_GRID[k + 1]
        mid = (lo + hi) / 2
        if m < mid or (m == mid and k % 2 == 0):
            return k
    return 7


def test_quarter_fold_gives_the_same_codes():
    """NVFP4 + H16 quantiser: the quotient is taken from w = 4v (the butterflies without
    their x0.25) and d' = 4d by the same FMA sequence. Where v = RN(w/4) is exactly w/4
    (|w| >= 2^-124), v/d and w/d' are one number, and wherever the sequence is exact
    (|v/d| >= 2^-3) both give RN(v/d). Every code, tiny quotients included, equals the
    code of RN(v/d), with w's sign. The block amax of v is RN(amax|w| / 4) because
    rounding is monotonic and odd."""
    rng = np.random.default_rng(11)
    scales = e4m3_values()
    tiny = Fraction(2) ** -124
    checked = 0
    for _ in range(300):
        S = exact(np.float32(2.0) ** rng.uniform(-60, 60) * rng.uniform(1, 2))
        d = rn32(scales[rng.integers(len(scales))] * S)
        e = 4 * d
        if not (Fraction(2) ** -100 <= e <= Fraction(2) ** 100):
            continue
        ws = [rn32(Fraction(float(rng.uniform(-32, 32))) * d) for _ in range(10)]
        ws += [Fraction(int(k)) * Fraction(2) ** -133 * 2 ** int(rng.integers(0, 12))
               for k in rng.integers(-127, 128, size=6)]  # bf16-subnormal-sized sums
        for w in ws:
            v = rn32(w / 4)
            folded = fma_sequence(w, e)
            plain = rn32(v / d)
            if abs(w) >= tiny and abs(plain) >= Fraction(1, 8):
                assert folded == plain, (w, d)
            assert e2m1_magnitude_code(abs(folded)) == e2m1_magnitude_code(abs(plain)), (w, d)
            assert folded == 0 or (folded < 0) == (w < 0)
            checked += 1
        block = ws[:16]
        assert rn32(max(abs(w) for w in block) / 4) == max(abs(rn32(w / 4)) for w in block)
    assert checked > 3000


# ---- IEEE signed zeros, for the sign-preserving form of the sequence ------------------
# A value is (x, neg): x a Fraction; neg is its sign bit (which matters only for x == 0).
def _val(x: Fraction, neg_zero: bool = False):
    return (x, (x < 0) if x != 0 else neg_zero)


def _neg(a):
    return (-a[0], not a[1])


def fma_rn(a, b, c):
    """RN(a*b + c) with IEEE zero signs: an exact zero sum is +0 unless both addends are
    -0; a nonzero result that rounds to zero keeps its sign."""
    prod = a[0] * b[0]
    prod_neg = (prod < 0) if prod != 0 else (a[1] != b[1])
    exact = prod + c[0]
    if exact != 0:
        r = rn32(exact)
        return (r, exact < 0) if r != 0 else (Fraction(0), exact < 0)
    if prod == 0 and c[0] == 0:
        return (Fraction(0), prod_neg and c[1])
    return (Fraction(0), False)  # cancellation of nonzero terms: +0


def mul_rn(a, b):
    """RN(a*b) with IEEE zero signs (a zero product's sign is the XOR of the operands')."""
    prod = a[0] * b[0]
    if prod != 0:
        r = rn32(prod)
        return (r, prod < 0)
    return (Fraction(0), a[1] != b[1])


def signed_sequence(v, e):
    """The quantiser's sign-preserving form: n = RN(q*e - v) (the negated residual), and
    each step q + (-n)*y, so that no sign copy is needed."""
    y = _val(rn32(1 / e[0]))
    nv = _neg(v)
    q0 = mul_rn(v, y)
    q1 = fma_rn(_neg(fma_rn(q0, e, nv)), y, q0)
    return fma_rn(_neg(fma_rn(q1, e, nv)), y, q1)


def test_signed_sequence_keeps_the_sign_and_the_code():
    """Without a sign copy, the sequence gives the quotient of v's sign (also for v = +-0
    and for quotients that underflow) and the same E2M1 code as RN(v/d); where the
    sequence is exact (|v/d| >= 2^-3) it gives RN(v/d) itself."""
    rng = np.random.default_rng(13)
    scales = e4m3_values()
    checked = 0
    for _ in range(300):
        S = exact(np.float32(2.0) ** rng.uniform(-60, 60) * rng.uniform(1, 2))
        d = rn32(scales[rng.integers(len(scales))] * S)
        e = 4 * d
        if not (Fraction(2) ** -100 <= e <= Fraction(2) ** 100):
            continue
        mags = [rn32(Fraction(float(rng.uniform(0, 32))) * d) for _ in range(8)]
        mags += [Fraction(int(k)) * Fraction(2) ** -133 * 2 ** int(rng.integers(0, 12))
                 for k in rng.integers(1, 128, size=6)]
        for m in mags:
            for neg in (False, True):
                w = -m if neg else m
                q, q_neg = signed_sequence(_val(w), _val(e))
                assert q_neg == neg, (w, e)
                plain = rn32(w / e)
                assert e2m1_magnitude_code(abs(q)) == e2m1_magnitude_code(abs(plain)), (w, e)
                if abs(plain) >= Fraction(1, 8):
                    assert q == plain, (w, e)
                checked += 1
        for neg in (False, True):  # signed zeros
            q, q_neg = signed_sequence(_val(Fraction(0), neg), _val(e))
            assert q == 0 and q_neg == neg
    assert checked > 5000
