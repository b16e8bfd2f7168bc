"""The correctly rounded division the quantisers use (csrc/beam_moe_div.cuh): x / d from
y = RN(1 / d), q0 = RN(x y), one FMA correction to bring q0 within an ulp, and Markstein's
final step (IBM J. Res. Develop. 34(1), 1990), whose exact remainder is asserted.  The steps
are restated here in exact rational arithmetic, rounding to binary32 after each operation as
the device does, and compared with the correctly rounded quotient on random and adversarial
operands over the range the quantisers use (d normal, quotients up to a few hundred).  The
device code itself is checked by the bit-exact E4M3 and NVFP4 quantisation tests."""
import random
from fractions import Fraction

import numpy as np
import pytest


def rn32(q: Fraction) -> Fraction:
    """q rounded to the nearest binary32 value, ties to even (no overflow in these tests)."""
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp = Fraction(2) ** max(e - 23, -149)
    n = a // ulp
    rem = a - n * ulp
    if rem * 2 > ulp or (rem * 2 == ulp and n % 2 == 1):
        n += 1
    return (1 if q > 0 else -1) * n * ulp


def f32(v: float) -> Fraction:
    return Fraction(float(np.float32(v)))


def div_rn_by(x: Fraction, d: Fraction) -> Fraction:
    y = rn32(1 / d)
    q0 = rn32(x * y)
    q1 = rn32(rn32(x - d * q0) * y + q0)
    assert abs(x / d - q1) < ulp32(q1), "the corrected quotient is within an ulp"
    rem = rn32(x - d * q1)
    assert rem == x - d * q1, "Markstein's remainder is exact"
    return rn32(rem * y + q1)


def ulp32(q: Fraction) -> Fraction:
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    return Fraction(2) ** max(e - 23, -149)


def _check(x, d):
    assert div_rn_by(x, d) == rn32(x / d), (float(x), float(d))


def test_random_operands_match_the_rounded_quotient():
    rng = random.Random(7)
    for _ in range(20000):
        d = f32(rng.uniform(1.0, 2.0) * 2.0 ** rng.randint(-90, 90))
        q = rng.uniform(-500.0, 500.0)
        x = f32(float(q * d))
        _check(x, d)


def test_bf16_dividends_and_e4m3_times_row_scales():
    # dividends with 8 significant bits (BF16), divisors s * value(bs) as the quantisers form
    rng = random.Random(11)
    e4m3 = [m * 2.0 ** e for e in range(-6, 9) for m in (1, 1.125, 1.25, 1.375, 1.5, 1.625, 1.75, 1.875)]
    for _ in range(20000):
        s = f32(rng.uniform(1.0, 2.0) * 2.0 ** rng.randint(-40, 10))
        d = rn32(s * f32(rng.choice(e4m3)))
        mant = rng.randint(128, 255) / 128.0
        x = f32(mant * float(d) * 2.0 ** rng.randint(-8, 2) * rng.choice((-1, 1)))
        bf = np.array([float(x)], np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
        x = Fraction(float(bf.view(np.float32)[0]))
        _check(x, d)


@pytest.mark.parametrize("k", [-60, -1, 0, 1, 37])
def test_adversarial_divisors(k):
    # divisors just below and above powers of two, where 1 / d rounds farthest
    for m in (1 - 2.0 ** -24, 1 + 2.0 ** -23, 1.5 - 2.0 ** -23, 1.75 + 2.0 ** -22):
        d = f32(m * 2.0 ** k)
        for x in (1.0, 3.0, 6.0, 448.0, 0.25, 5.0, 2688.0, 1 + 2.0 ** -7, 255.0 / 128):
            for sx in (1, -1):
                _check(f32(sx * x * float(d) * (1 + 2.0 ** -20)), d)
                _check(f32(sx * x), d)
