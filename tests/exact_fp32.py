"""Exact rational arithmetic with IEEE-754 binary32 round-to-nearest-even.

Used to pin the oracle's fp32 evaluation order against the mathematics of
correctly rounded fp32 operations, independently of any C library or
compiler: every result is the exact rational value rounded once.
"""
from fractions import Fraction

import numpy as np

_MAX = Fraction((2 ** 24 - 1) * 2 ** 104)


def f(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def round_f32(x: Fraction) -> Fraction:
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp_e = max(e - 23, -149)
    scaled = a / Fraction(2) ** ulp_e
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = n * Fraction(2) ** ulp_e
    if r > _MAX:
        raise OverflowError
    return sign * r


def fma32(a: Fraction, b: Fraction, c: Fraction) -> Fraction:
    return round_f32(a * b + c)


def add32(a: Fraction, b: Fraction) -> Fraction:
    return round_f32(a + b)


def mul32(a: Fraction, b: Fraction) -> Fraction:
    return round_f32(a * b)
