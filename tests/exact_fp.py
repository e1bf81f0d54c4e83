"""Exact rational IEEE-754 rounding (round to nearest, ties to even), written
from the definition: the independent route the oracle pins use to check
NumPy's fp32 arithmetic and its fp32 -> fp16 casts."""

from fractions import Fraction

FP32 = (24, -126, 127)   # significand bits (with the hidden bit), emin, emax
FP16 = (11, -14, 15)


def round_to_format(value: Fraction, fmt) -> Fraction:
    mant, emin, emax = fmt
    if value == 0:
        return Fraction(0)
    sign = -1 if value < 0 else 1
    a = abs(value)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)                       # subnormals share emin's quantum
    quantum = Fraction(2) ** (e - mant + 1)
    r = round(a / quantum)                 # Fraction rounding: half to even
    val = r * quantum
    if val >= Fraction(2) ** (emax + 1):
        return Fraction(sign) * Fraction(10**400)   # stands for infinity
    return sign * val


def rn32(v) -> Fraction:
    """The fp32 value nearest to v (ties to even)."""
    return round_to_format(Fraction(v), FP32)


def rn16(v) -> Fraction:
    """The fp16 value nearest to v (ties to even); 10**400 stands for +inf."""
    return round_to_format(Fraction(v), FP16)


BF16 = (8, -126, 127)
