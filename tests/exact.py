"""Exact rational arithmetic used to pin the oracle (test-side only).

Everything here works on ``fractions.Fraction`` values, so it carries no
floating-point rounding at all; it restates definitions (nearest value of a
format, nearest grid point) by search or exact comparison, never by calling
the oracle.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np


def f16_value(bits: int) -> Fraction:
    """Exact value of a finite binary16 bit pattern (IEEE 754 definition)."""
    s = -1 if bits >> 15 else 1
    e = (bits >> 10) & 0x1F
    m = bits & 0x3FF
    assert e != 31, "not finite"
    if e == 0:
        return s * Fraction(m, 1 << 24)
    return s * Fraction(m | 0x400, 1) * Fraction(2) ** (e - 25)


ALL_FINITE_F16 = np.array([b for b in range(1 << 16) if ((b >> 10) & 0x1F) != 31], dtype=np.uint16)
# positive finite values in increasing order, with +0
POS_F16 = np.array([b for b in range(0, 0x7C00)], dtype=np.uint16)


def round_half_even(v: Fraction) -> int:
    fl = math.floor(v)
    d = v - fl
    if d > Fraction(1, 2):
        return fl + 1
    if d < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def nearest_f16_bits(v: Fraction) -> int:
    """Nearest binary16 to a non-negative finite rational by bisection over the
    ordered positive bit patterns (ties -> even fraction bit), or 0x7C00 when
    it lies at or beyond the overflow midpoint."""
    assert v >= 0
    maxf = f16_value(0x7BFF)
    if v >= maxf + (Fraction(2) ** 15 - maxf) / 2:   # midpoint toward 2^16
        return 0x7C00
    lo, hi = 0, 0x7BFF
    # largest pattern with value <= v
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if f16_value(mid) <= v:
            lo = mid
        else:
            hi = mid - 1
    a = lo
    if f16_value(a) == v or a == 0x7BFF:
        return a
    b = a + 1
    da, db = v - f16_value(a), f16_value(b) - v
    if da < db:
        return a
    if db < da:
        return b
    return a if a % 2 == 0 else b
