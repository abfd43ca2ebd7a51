"""Exact rational arithmetic helpers for pinning the oracle.

These are written from the IEEE 754 definition of round-to-nearest-even and
share nothing with the oracle's C code: values are Python Fractions and the
rounding is done by integer arithmetic on the exact value.
"""
from __future__ import annotations

import struct
from fractions import Fraction


def f32(x: float) -> float:
    """Round a Python float (binary64) to binary32 and back (numpy-free)."""
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0]


def bits_f32(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", b & 0xFFFFFFFF))[0]


def _floor_log2(a: Fraction) -> int:
    """floor(log2(a)) for a > 0, exactly."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    # now 2^(e-1) < a < 2^(e+1); fix up
    if a >= Fraction(2) ** e:
        while a >= Fraction(2) ** (e + 1):
            e += 1
    else:
        while a < Fraction(2) ** e:
            e -= 1
    return e


def round_rne(v: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round an exact value to the binary format with `mant_bits` significand
    bits (hidden bit included) and minimum normal exponent `emin`, ties to
    even.  No overflow handling (callers stay in range)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = max(_floor_log2(a), emin)
    ulp = Fraction(2) ** (e - (mant_bits - 1))
    q = a / ulp
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * ulp


def to_f32(v: Fraction) -> float:
    """Exact value -> nearest binary32 (ties to even) as a Python float."""
    return float(round_rne(v, 24, -126))


def to_bf16(v: Fraction) -> float:
    """Exact value -> nearest bfloat16 (ties to even) as a Python float."""
    return float(round_rne(v, 8, -126))


def bf16_bits(x: float) -> int:
    """Bit pattern of a value already representable in bf16."""
    b = f32_bits(x)
    assert b & 0xFFFF == 0, "value is not a bf16"
    return b >> 16
