"""Exact-rational reference arithmetic used to pin the oracle.

Everything here works on ``fractions.Fraction`` from the bit fields of each
format, independently of the oracle's numpy implementation, so a slip in the
oracle (a wrong bias, a dropped rounding case, a wrong group index) shows up as
a disagreement with these functions.
"""

from __future__ import annotations

from fractions import Fraction

HALF = Fraction(1, 2)


def pow2(e: int) -> Fraction:
    return Fraction(2) ** e


def bf16_value(bits: int):
    """BF16 bits -> Fraction (or the strings 'nan', '+inf', '-inf')."""
    s = (bits >> 15) & 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0xFF:
        return "nan" if m else ("-inf" if s else "+inf")
    v = Fraction(m, 128) * pow2(-126) if e == 0 else (1 + Fraction(m, 128)) * pow2(e - 127)
    return -v if s else v


def e4m3_value(b: int):
    """OCP E4M3 byte -> Fraction (or 'nan')."""
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 0x7
    if e == 0xF and m == 0x7:
        return "nan"
    v = Fraction(m, 8) * pow2(-6) if e == 0 else (1 + Fraction(m, 8)) * pow2(e - 7)
    return -v if s else v


# E2M1 magnitudes as listed in the OCP MX v1.0 specification, by code & 7.
E2M1_MAGNITUDES = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2),
                   Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def e2m1_value(c: int) -> Fraction:
    v = E2M1_MAGNITUDES[c & 7]
    return -v if c & 8 else v


def fp32_value(bits: int) -> Fraction:
    s = (bits >> 31) & 1
    e = (bits >> 23) & 0xFF
    m = bits & 0x7FFFFF
    assert e != 0xFF
    v = Fraction(m, 1 << 23) * pow2(-126) if e == 0 else (1 + Fraction(m, 1 << 23)) * pow2(e - 127)
    return -v if s else v


def _exponent(a: Fraction) -> int:
    """e with 2**e <= a < 2**(e+1), for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while pow2(e) > a:
        e -= 1
    while pow2(e + 1) <= a:
        e += 1
    return e


def round_half_even(t: Fraction) -> int:
    n = t.numerator // t.denominator
    rem = t - n
    if rem > HALF or (rem == HALF and n % 2 == 1):
        n += 1
    return n


def bf16_bits_of(r: Fraction, negative_zero: bool = False) -> int:
    """Round an exact rational to BF16 (RNE) and encode the result's bits."""
    if r == 0:
        return 0x8000 if negative_zero else 0
    sign = 0x8000 if r < 0 else 0
    a = abs(r)
    e = _exponent(a)
    quantum = pow2(-133) if e < -126 else pow2(e - 7)
    v = round_half_even(a / quantum) * quantum
    if v == 0:
        return sign
    if v >= pow2(128):
        return sign | 0x7F80
    if v < pow2(-126):
        return sign | int(v / pow2(-133))
    ev = _exponent(v)
    mant = (v / pow2(ev) - 1) * 128
    assert mant.denominator == 1
    return sign | ((ev + 127) << 7) | int(mant)
