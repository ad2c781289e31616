"""The quantised dispatches take x / s as Markstein's correction from one
reciprocal per scale block (q0 = RN(x * r), the remainder x - q0*s, then
RN(q0 + rem * r), with r = RN(1 / s)).  This checks, in exact rational
arithmetic on the CPU, that the method returns the correctly rounded fp32
quotient over the range the kernels use it in (s in [2^-60, 2^60]; |x / s|
at most 448), so that taking it instead of a division changes no bit."""

from fractions import Fraction

import numpy as np
import pytest

F32 = np.float32


def rn32(q: Fraction) -> np.float32:
    """Round an exact rational to the nearest fp32, ties to even."""
    c = F32(float(q))  # within one fp32 step of the answer
    cands = {c, np.nextafter(c, F32(np.inf)), np.nextafter(c, F32(-np.inf))}
    best = min(cands, key=lambda v: (abs(Fraction(float(v)) - q),
                                     int(np.array(v, F32).view(np.uint32)) & 1))
    return F32(best)


def fma32(a, b, c) -> np.float32:
    """fp32 fused multiply-add: a*b + c exactly, rounded once."""
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def markstein(x, s, r):
    q0 = rn32(Fraction(float(x)) * Fraction(float(r)))
    rem = fma32(-q0, s, x)
    q = fma32(rem, r, q0)
    return F32(np.copysign(q, x))


def _cases(rng, n):
    s = (rng.uniform(1.0, 2.0, n) * 2.0 ** rng.integers(-60, 60, n)).astype(F32)
    q = rng.uniform(-448.0, 448.0, n)
    x = (q * s.astype(np.float64)).astype(F32)
    return x, s


def test_markstein_quotient_is_correctly_rounded():
    rng = np.random.default_rng(16)
    x, s = _cases(rng, 4000)
    # quotients near fp32 rounding boundaries: x = s * (a value one step off a midpoint)
    mids = (rng.uniform(1, 448, 500).astype(F32)).astype(np.float64)
    s2 = (rng.uniform(1.0, 2.0, 500) * 2.0 ** rng.integers(-20, 20, 500)).astype(F32)
    x2 = (mids * s2.astype(np.float64)).astype(F32)
    x, s = np.concatenate([x, x2]), np.concatenate([s, s2])
    for xi, si in zip(x, s):
        ri = rn32(1 / Fraction(float(si)))
        want = rn32(Fraction(float(xi)) / Fraction(float(si)))
        got = markstein(xi, si, ri)
        assert np.array(got, F32).view(np.uint32) == np.array(want, F32).view(np.uint32), (xi, si)


@pytest.mark.parametrize("x", [0.0, -0.0])
def test_markstein_keeps_the_sign_of_zero(x):
    s = F32(0.37)
    r = rn32(1 / Fraction(float(s)))
    got = markstein(F32(x), s, r)
    assert got == 0 and np.signbit(got) == np.signbit(F32(x))


def test_tiny_quotients_stay_below_the_e4m3_and_e2m1_zero_thresholds():
    """Below |x / s| = 2^-12 the result need not be the rounded quotient,
    but it stays below 2^-11 with the sign of x, which every e4m3 and e2m1
    encoding maps to the same signed zero."""
    rng = np.random.default_rng(3)
    for _ in range(2000):
        s = F32(rng.uniform(1, 2) * 2.0 ** rng.integers(-60, 60))
        x = F32(rng.uniform(-1, 1) * 2.0 ** -12 * float(s) * 2.0 ** -float(rng.integers(0, 40)))
        r = rn32(1 / Fraction(float(s)))
        got = markstein(x, s, r)
        assert abs(float(got)) < 2.0 ** -11
        assert got == 0 or np.signbit(got) == np.signbit(x)
