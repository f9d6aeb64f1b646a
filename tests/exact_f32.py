"""Exact binary32 arithmetic for pinning the oracle: every operation is carried out on exact rationals
(Python `fractions`) and rounded once to the nearest binary32 (ties to even, gradual underflow), the way
IEEE 754 defines a correctly rounded operation.  A fused multiply-add is the exact a*b + c rounded once.
Test infrastructure only; independent of the oracle's C code and of the CUDA path."""
from __future__ import annotations

from fractions import Fraction

import numpy as np

EMIN = -126          # smallest normal exponent of binary32
P = 24               # significand bits
MAX = Fraction(2 ** P - 1, 2 ** (P - 1)) * 2 ** 127


def rne(q: Fraction) -> Fraction:
    """The binary32 value nearest to q (ties to even); +-inf past the overflow threshold."""
    if q == 0:
        return Fraction(0)
    s = -1 if q < 0 else 1
    a = -q if q < 0 else q
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, EMIN) - (P - 1))
    m = a / quantum
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = lo * quantum
    if v > MAX:
        return Fraction(s) * Fraction(10) ** 400   # stands for infinity (never reached by the pins)
    return s * v


def to_f32(q: Fraction) -> np.float32:
    return np.float32(float(rne(q)))


def f(x) -> Fraction:
    """Exact rational value of a binary32 (or binary64) number."""
    return Fraction(float(x))


def mul(a: Fraction, b: Fraction) -> Fraction:
    return rne(a * b)


def add(a: Fraction, b: Fraction) -> Fraction:
    return rne(a + b)


def fma(a: Fraction, b: Fraction, c: Fraction) -> Fraction:
    return rne(a * b + c)


def rint_even(q: Fraction) -> int:
    """Round to the nearest integer, ties to even (rintf in the default rounding mode)."""
    lo = q.numerator // q.denominator
    rem = q - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return lo
