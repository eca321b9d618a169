"""Exact-rational helpers for brute-force checks of the oracle (tests only).

Rounding to binary32 / bf16 is done on ``fractions.Fraction`` values with a
single round-to-nearest-even step, so it does not rely on fp64 intermediates.
"""

from fractions import Fraction

import numpy as np

HALF = Fraction(1, 2)


def _floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    return e


def round_to_precision(v: Fraction, sig_bits: int, min_exp: int) -> Fraction:
    """Nearest (ties-to-even) binary number with ``sig_bits`` significant bits;
    below 2**min_exp the quantum is fixed (gradual underflow)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = max(_floor_log2(a), min_exp)
    quantum = Fraction(2) ** (e - (sig_bits - 1))
    m = a / quantum
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > HALF or (rem == HALF and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def rn32(v: Fraction) -> Fraction:
    return round_to_precision(v, 24, -126)


def rn_bf16(v: Fraction) -> Fraction:
    return round_to_precision(v, 8, -126)


def rne_int(v: Fraction) -> int:
    fl = v.numerator // v.denominator
    rem = v - fl
    if rem > HALF or (rem == HALF and fl % 2 == 1):
        fl += 1
    return fl


def frac(x) -> Fraction:
    return Fraction(float(x))


def f32_bits_of(v: Fraction) -> int:
    return int(np.float32(float(v)).view(np.uint32))
