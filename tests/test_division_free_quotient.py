"""The identity the quantize+pack kernel relies on instead of a division:
with r = RN(1/s), d = RN(x - m), q0 = RN(d r), e = RN(d - q0 s) (one fma,
exact) and q1 = RN(q0 + e r) (one fma), q1 == RN(d / s) (Markstein's
correction step), hence rint(q1) is the defined code rint(RN(d / s)).

Checked in exact rational arithmetic with fp32 round-to-nearest-even written
out, on cells drawn as the quantizer meets them (bf16 min and max, s from the
definition) and on values placed at and next to half-integer quotients,
for every bit width.  No GPU, no oracle: a property of the arithmetic."""
import random
from fractions import Fraction

import pytest


def rn32(x: Fraction) -> Fraction:
    """fp32 round-to-nearest-even of a rational (normal and subnormal range)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    q, rem = divmod(a, ulp)
    q = int(q)
    if rem > ulp / 2 or (rem == ulp / 2 and q % 2 == 1):
        q += 1
    return sign * q * ulp


def bf16(x: float) -> Fraction:
    """A bf16 value near x (round to nearest, 8 significant bits)."""
    f = Fraction(x)
    if f == 0:
        return f
    e = abs(f).numerator.bit_length() - abs(f).denominator.bit_length()
    ulp = Fraction(2) ** (e - 8)
    return round(f / ulp) * ulp


def rint_even(x: Fraction) -> int:
    q, rem = divmod(x, 1)
    q = int(q)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1):
        q += 1
    return q


def division_free(x, m, s, r):
    d = rn32(x - m)
    q0 = rn32(d * r)
    e = rn32(d - q0 * s)
    q1 = rn32(q0 + e * r)
    return q1, rn32(d / s)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_quotient_matches_division(bits):
    rng = random.Random(bits)
    qmax = (1 << bits) - 1
    checked = ties = 0
    for _ in range(60):
        lo = rng.choice([-80.0, -3.0, -0.05, 0.0, 1.5, 1000.0]) * rng.uniform(0.5, 2.0)
        hi = lo + rng.choice([1e-3, 0.7, 5.0, 160.0, 3e4]) * rng.uniform(0.5, 2.0)
        m, mx = bf16(lo), bf16(hi)
        if mx <= m:
            continue
        s = rn32(rn32(mx - m) / qmax)
        r = rn32(1 / s)
        xs = [bf16(float(m + (mx - m) * rng.random())) for _ in range(40)]
        # values at and next to half-integer quotients: m + (k + 1/2) s on the bf16 grid
        for k in range(qmax):
            t = m + (k + Fraction(1, 2)) * s
            b = bf16(float(t))
            e = abs(b).numerator.bit_length() - abs(b).denominator.bit_length() if b != 0 else -126
            ulp = Fraction(2) ** (e - 8)
            xs += [b - ulp, b, b + ulp]
        for x in xs:
            if x < m or x > mx:
                continue
            q1, q = division_free(x, m, s, r)
            assert q1 == q, (bits, float(x), float(m), float(s))
            assert rint_even(q1) == rint_even(q)
            checked += 1
            ties += q.denominator == 2
    assert checked > 1000
