"""Exact-arithmetic models used to pin the oracle: rational numbers rounded to
IEEE binary32 / bfloat16 by round-to-nearest-even, written from the format
definitions (independent of C's fmaf, of numpy and of torch)."""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def _round(v: Fraction, sig_bits: int, emin: int, emax: int) -> Fraction:
    """Round to a binary format with `sig_bits` significant bits (incl. the implicit
    one), minimum normal exponent emin and maximum exponent emax; ties to even."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, emin) - (sig_bits - 1))
    n = a / quantum
    q = n.numerator // n.denominator
    rem = n - q
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1):
        q += 1
    r = q * quantum
    if r >= Fraction(2) ** (emax + 1):
        raise OverflowError
    return sign * r


def f32(v: Fraction) -> Fraction:
    return _round(v, 24, -126, 127)


def bf16(v: Fraction) -> Fraction:
    return _round(v, 8, -126, 127)


def fmaf(a, b, c) -> Fraction:
    return f32(Fraction(a) * Fraction(b) + Fraction(c))


def addf(a, b) -> Fraction:
    return f32(Fraction(a) + Fraction(b))


def to_float32(v: Fraction) -> np.float32:
    return np.float32(float(v))          # exact: v is a binary32 value


def bf16_bits(v: Fraction) -> int:
    f = np.array([float(v)], dtype=np.float32)
    return int(f.view(np.uint32)[0] >> 16)


def bf16_value(bits: int) -> Fraction:
    f = np.array([int(bits) << 16], dtype=np.uint32).view(np.float32)[0]
    return Fraction(float(f))
