"""Exact rational helpers for brute-force pins (tests only).

rn32 rounds a rational to the nearest IEEE fp32 value (ties to even) with integer
arithmetic, so that a test can evaluate an fp32 recipe step by step without
trusting any floating-point unit.  Normal-range values only."""
from fractions import Fraction

import numpy as np


def rne_int(x: Fraction) -> int:
    """Round a rational to the nearest integer, ties to even (torch.round)."""
    n = x.numerator // x.denominator          # floor
    r = x - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def _rn_bits(x: Fraction, sig_bits: int) -> Fraction:
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - (sig_bits - 1))
    return sign * rne_int(a / ulp) * ulp


def rn32(x: Fraction) -> Fraction:
    """Nearest fp32 value (24 significant bits), ties to even; normal range assumed."""
    v = _rn_bits(x, 24)
    if v != 0:
        assert Fraction(2) ** -126 <= abs(v) < Fraction(2) ** 128, "outside fp32 normal range"
    return v


def rn_bf16(x: Fraction) -> Fraction:
    """Nearest bf16 value (8 significant bits), ties to even."""
    return _rn_bits(x, 8)


def f32(x) -> Fraction:
    """Exact rational value of an fp32 number."""
    return Fraction(float(np.float32(x)))


def bf16_bits_to_fraction(b: int) -> Fraction:
    return Fraction(float(np.array([int(b) << 16], np.uint32).view(np.float32)[0]))
