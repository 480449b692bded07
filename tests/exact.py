"""Exact-rational restatements of IEEE-754 rounding, used to pin the oracle.

Everything here works on ``fractions.Fraction`` values, so it shares no
floating-point code with numpy or with the oracle: a binary format is rounded
to nearest, ties to even, by looking at the exact quotient.
"""
from __future__ import annotations

from fractions import Fraction
import math

import numpy as np

INF = float("inf")


def _floor_log2(a: Fraction) -> int:
    """floor(log2(a)) for a > 0, exactly."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    # 2^e <= a < 2^(e+1) after at most one correction
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def round_binary(x: Fraction, p: int, emin: int, emax: int):
    """Round x to the binary format with p significand bits (incl. hidden),
    minimum normal exponent emin and maximum exponent emax; round half to
    even; overflow gives +-inf. Returns a Fraction or +-inf."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = max(_floor_log2(a), emin)
    ulp = Fraction(2) ** (e - (p - 1))
    n = round(a / ulp)          # Fraction.__round__ is round-half-even
    r = n * ulp
    if r >= Fraction(2) ** (emax + 1):
        return sign * INF
    return sign * r


def fp32(x: Fraction):
    return round_binary(x, 24, -126, 127)


def fp16(x: Fraction):
    return round_binary(x, 11, -14, 15)


def frac(v) -> Fraction:
    """Exact value of a finite numpy/python float."""
    return Fraction(float(v))


def round_half_even(x: Fraction) -> int:
    return round(x)


def to_f16_bits(v) -> int:
    """Bit pattern of an exact value that is representable in binary16."""
    if v in (INF, -INF):
        return 0x7C00 | (0x8000 if v < 0 else 0)
    return int(np.float16(float(v)).view(np.uint16)) if v != 0 else 0


def div_rne_exact(a: int, b: int) -> int:
    """Round-half-even of the exact rational a/b (b != 0)."""
    return round(Fraction(a, b))


assert math.isinf(INF)
