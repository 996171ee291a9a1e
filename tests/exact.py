"""Exact-rational reference arithmetic for pinning the oracle (no numpy rounding involved).

fp16 rounding is written out from the IEEE binary16 format itself: 11 significant bits, minimum
normal exponent -14, subnormal quantum 2^-24, ties to even, overflow above 65504 + 16 to inf.
"""
from __future__ import annotations

import math
from fractions import Fraction

FP16_MAX = Fraction(65504)


def round_half_even(x: Fraction) -> int:
    """Nearest integer to x, ties to the even integer."""
    fl = math.floor(x)
    rem = x - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def fp16_quantum(x: Fraction) -> Fraction:
    """Spacing of the binary16 grid around |x| (x != 0)."""
    ax = abs(x)
    if ax < Fraction(1, 2 ** 14):
        return Fraction(1, 2 ** 24)
    e = ax.numerator.bit_length() - ax.denominator.bit_length()
    if Fraction(2) ** e > ax:          # make 2^e <= ax < 2^(e+1)
        e -= 1
    elif Fraction(2) ** (e + 1) <= ax:
        e += 1
    return Fraction(2) ** (e - 10)


def fp16_round_exact(x: Fraction) -> Fraction | float:
    """Correctly rounded binary16 value of the exact rational x (float('inf') on overflow)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    ax = abs(x)
    qn = fp16_quantum(ax)
    r = round_half_even(ax / qn) * qn
    if r > FP16_MAX:
        return sign * float("inf")
    return sign * r


def code_exact(x: Fraction, s: Fraction, z: Fraction, bits: int) -> int:
    """Q of one element with exact arithmetic: clamp(RNE((x - z)/s), 0, 2^b - 1); s == 0 -> 0."""
    if s == 0:
        return 0
    return min(max(round_half_even((x - z) / s), 0), 2 ** bits - 1)


def code_nearest_grid(x: Fraction, s: Fraction, z: Fraction, bits: int) -> int:
    """Q found by search instead of division: the grid point z + k*s (k = 0..2^b-1) nearest to x,
    ties to the even k.  Equal to code_exact whenever s > 0."""
    best = None
    for k in range(2 ** bits):
        dist = abs(x - (z + k * s))
        if best is None or dist < best[0] or (dist == best[0] and k % 2 == 0):
            best = (dist, k)
    return best[1]
