"""Exact rational helpers for the oracle's pins (tests only).

Rounds rationals to binary floating point by integer arithmetic, so that a
pin does not reuse numpy's or the oracle's float conversions.
"""

from fractions import Fraction


def _floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def round_nearest_even(x: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round to the nearest binary float with ``mant_bits`` fraction bits and
    minimum normal exponent ``emin`` (subnormals kept), ties to even."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = max(_floor_log2(a), emin)
    quantum = Fraction(2) ** (e - mant_bits)
    scaled = a / quantum
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * lo * quantum


def rn_f32(x: Fraction) -> Fraction:
    return round_nearest_even(x, 23, -126)


def rn_bf16(x: Fraction) -> Fraction:
    return round_nearest_even(x, 7, -126)


def frac(v) -> Fraction:
    """Exact rational value of a Python/numpy float."""
    return Fraction(float(v))
