"""Exact rational arithmetic used to pin the oracle independently of its C code.

Nothing here uses the oracle's floating-point evaluation order: values are
carried as :class:`fractions.Fraction` and rounded once, correctly, to the
target format.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def round_half_even(v: Fraction) -> int:
    """Nearest integer to a rational, ties to even."""
    fl = math.floor(v)
    rem = v - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def to_fp32(v: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 value of a rational.

    Handles normal numbers only (the pins never reach the subnormal range)."""
    if v == 0:
        return np.float32(0.0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix the estimate so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    m = round_half_even(a * Fraction(2) ** (23 - e))  # 24-bit significand
    if m == 2 ** 24:
        m, e = 2 ** 23, e + 1
    return np.float32(sign * m * 2.0 ** (e - 23))


def fr(x) -> Fraction:
    """Exact rational value of a float (numpy or Python)."""
    return Fraction(float(x))


def bf16_bits(values) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable in bf16."""
    f = np.asarray(values, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the bits."""
    u = np.asarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def exact_to_bf16_bits(v: Fraction) -> int:
    """Round an exact rational once, to nearest with ties to even, to bfloat16
    (8 significant bits, fp32's exponent range); returns the bit pattern."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = -v if v < 0 else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if e < -126:
        q = Fraction(1, 2 ** 133)
    else:
        q = Fraction(2) ** (e - 7)
    n = round_half_even(a / q)
    r = n * q
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80
    f = np.float32(float(r))  # exact: at most 8 significant bits
    return sign | int((f.view(np.uint32) >> 16) & 0x7FFF)
