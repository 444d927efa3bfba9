"""The quantisers' shared-divisor division, checked as a method on the host.

The e4m3 / NVFP4 codes are decided by fp32 quotients x / scale rounded to nearest
(the oracle divides in IEEE fp32).  The kernels compute them as y = RN(1/s),
q = RN(x*y), then two of Markstein's correction steps q <- RN(q + RN(x - s*q)*y),
each residual formed by one FMA (csrc/quant_div.cuh).  This test runs that
sequence in exact rational arithmetic, with every fp32 rounding done explicitly,
and compares it with the exactly rounded quotient: random pairs over the ranges
the quantisers see, and pairs whose quotient lies within a few units of the last
place of a rounding midpoint (where a single uncorrected product fails).  It pins
the method independently of the GPU; the device function is compared with CUDA's
IEEE division bit for bit by a GPU test.
"""
from fractions import Fraction

import numpy as np
import pytest


def rn32(v: Fraction) -> Fraction:
    """Round a rational to the nearest fp32 value (ties to even), as an exact rational;
    overflow is not reached by the inputs used here."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                       # subnormal range: quantum 2^-149
    quantum = Fraction(2) ** (e - 23)
    n, rem = divmod(a, quantum)
    n = int(n)
    half = quantum / 2
    if rem > half or (rem == half and n % 2 == 1):
        n += 1
    return sign * n * quantum


def fma32(a: Fraction, b: Fraction, c: Fraction) -> Fraction:
    return rn32(a * b + c)


def div_markstein(x: Fraction, s: Fraction) -> Fraction:
    y = rn32(1 / s)
    q = rn32(x * y)
    for _ in range(2):
        r = fma32(-q, s, x)
        q = fma32(r, y, q)
    return q


def f32(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def _pairs(n, seed):
    rng = np.random.default_rng(seed)
    # divisors: scales amax/448 and NVFP4 block scales over a wide range; dividends
    # up to 448 times the divisor, as in the quantisers, plus arbitrary ones
    s = (rng.uniform(1.0, 2.0, n) * np.exp2(rng.integers(-60, 40, n))).astype(np.float32)
    t = rng.uniform(-448.0, 448.0, n).astype(np.float64)
    x = (t * s.astype(np.float64)).astype(np.float32)
    return x, s


def test_random_pairs_round_correctly():
    x, s = _pairs(4000, 1)
    for xi, si in zip(x, s):
        X, S = f32(xi), f32(si)
        assert div_markstein(X, S) == rn32(X / S), (float(xi), float(si))


def test_near_midpoint_quotients_round_correctly():
    """Quotients within +-3 units of 2^-30 of an fp32 rounding midpoint, in the
    binades that decide e4m3 and e2m1 codes; the uncorrected RN(x * RN(1/s)) is
    wrong on a good share of them, the corrected quotient on none."""
    rng = np.random.default_rng(7)
    wrong_single = 0
    cases = 0
    for _ in range(3000):
        S = f32(np.float32(rng.uniform(1.0, 2.0) * 2.0 ** int(rng.integers(-40, 30))))
        e = int(rng.integers(-11, 9))
        m = int(rng.integers(2 ** 23, 2 ** 24))
        mid = (Fraction(m) + Fraction(1, 2)) * Fraction(2) ** (e - 23)      # an fp32 midpoint
        for k in (-3, -1, 0, 1, 3):
            target = mid + k * Fraction(2) ** (e - 23 - 30)
            X = rn32(target * S)
            if X == 0:
                continue
            cases += 1
            exact = rn32(X / S)
            assert div_markstein(X, S) == exact, (float(X), float(S))
            wrong_single += rn32(X * rn32(1 / S)) != exact
    assert cases > 10000
    assert wrong_single > 0          # the cases do exercise the correction


def test_signed_zero_and_sign():
    S = f32(0.37)
    assert div_markstein(Fraction(0), S) == 0
    X = f32(-1.5)
    assert div_markstein(X, S) == rn32(X / S) < 0


@pytest.mark.parametrize("s", [448.0, 6.0 * 448.0])
def test_scale_constants(s):
    """amax / 448 (e4m3 scale) for amax over the bf16 grid around typical magnitudes."""
    rng = np.random.default_rng(3)
    S = Fraction(s)
    for a in rng.uniform(0.01, 64.0, 2000).astype(np.float32):
        A = f32(a)
        assert div_markstein(A, S) == rn32(A / S)
