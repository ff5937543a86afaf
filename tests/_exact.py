"""Exact rational arithmetic helpers for pinning the oracle.

These do not reuse the oracle's code: values are Python Fractions and the BF16
rounding below is derived from the format definition (1 sign, 8 exponent, 7
stored mantissa bits; subnormal quantum 2**-133), rounding half to even.
"""
from fractions import Fraction
import struct


def bf16_bits_to_fraction(bits: int) -> Fraction:
    f = struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]
    return Fraction(f)


def fraction_to_bf16_bits(v: Fraction) -> int:
    """Round an exact rational to the nearest BF16 (ties to even); finite range only."""
    if v == 0:
        return 0
    neg = v < 0
    a = -v if neg else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q_exp = max(e, -126) - 7          # quantum: 7 fractional mantissa bits
    m = a / (Fraction(2) ** q_exp)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    value = Fraction(fl) * (Fraction(2) ** q_exp)
    f32 = struct.unpack("<I", struct.pack("<f", float(value)))[0]
    assert Fraction(struct.unpack("<f", struct.pack("<I", f32))[0]) == value
    bits = f32 >> 16
    assert (f32 & 0xFFFF) == 0
    return bits | (0x8000 if neg else 0)


def round_half_even(v: Fraction) -> int:
    fl = v.numerator // v.denominator
    rem = v - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl
