"""Exact rational helpers for pinning the oracle (test code; independent of the oracle).

fp16 values are all integer multiples of 2^-24, so scaled by 2^24 they are exact
integers; rounding a rational to fp16 is done here from the IEEE 754 binary16
definition (10 fraction bits, minimum normal exponent -14, subnormal quantum
2^-24), not with numpy's float16 conversion.
"""
from fractions import Fraction

import numpy as np

Q24 = 1 << 24  # 2^24: one fp16 subnormal quantum is 1/Q24


def fp16_to_fraction(h) -> Fraction:
    bits = int(np.asarray(h, dtype=np.float16).view(np.uint16))
    sign = -1 if bits & 0x8000 else 1
    exp = (bits >> 10) & 0x1F
    man = bits & 0x3FF
    assert exp != 0x1F, "finite values only"
    if exp == 0:
        mag = Fraction(man, Q24)
    else:
        mag = Fraction(1024 + man, 1 << 10) * (Fraction(2) ** (exp - 15))
    return sign * mag


def round_half_even(fr: Fraction) -> int:
    fl = fr.numerator // fr.denominator
    rem = fr - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def fraction_to_fp16(fr: Fraction) -> np.float16:
    """Correctly rounded (RNE) binary16 value of an exact rational (no overflow handling)."""
    if fr == 0:
        return np.float16(0.0)
    sign = -1 if fr < 0 else 1
    x = abs(fr)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    while Fraction(2) ** (e + 1) <= x:
        e += 1
    e = max(e, -14)                       # below 2^-14 the quantum stays 2^-24
    quantum = Fraction(2) ** (e - 10)
    n = round_half_even(x / quantum)
    val = n * quantum
    assert val <= 65504
    return np.float16(sign * float(val))  # val has <= 11 significant bits: exact


def positive_fp16_values() -> np.ndarray:
    """All finite positive binary16 values, ascending (subnormals included)."""
    return np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)
