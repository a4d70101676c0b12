"""Exact-rational reference arithmetic for pinning the oracle.

Everything here works on ``fractions.Fraction`` values and is written from the number
formats' definitions (IEEE binary32, E4M3, E2M1): it never calls the oracle and shares no
code with it, so a test that compares the two checks the oracle against the mathematics.
"""
from __future__ import annotations

import struct
from fractions import Fraction as F

U = F(1, 2**24)                      # unit roundoff of binary32
FLT_MAX = F((2**24 - 1) * 2**104)

# E2M1 magnitudes by 3-bit index (Four Over Six, Problem definition)
E2M1_GRID = [F(0), F(1, 2), F(1), F(3, 2), F(2), F(3), F(4), F(6)]


def e4m3_values():
    """All non-negative finite E4M3 values, by code 0x00..0x7E (bias 7, 3 mantissa bits)."""
    out = []
    for code in range(0x7F):
        e, m = code >> 3, code & 7
        if e == 0:
            out.append(F(m, 8) * F(1, 2**6))
        else:
            out.append((1 + F(m, 8)) * (F(2) ** (e - 7)))
    return out


E4M3 = e4m3_values()


def f32_value(x: float) -> F:
    """Exact value of a binary32 (given as a Python float holding a binary32 value)."""
    return F(struct.unpack("<f", struct.pack("<f", x))[0])


def is_f32(v: F) -> bool:
    """True if v is exactly representable in binary32 (finite, subnormals included)."""
    if v == 0:
        return True
    a = abs(v)
    if a > FLT_MAX:
        return False
    # a = n / 2^k with n odd, or integer times power of two
    num, den = a.numerator, a.denominator
    if den & (den - 1):
        return False                      # denominator not a power of two
    # strip factors of two from the numerator
    tz = (num & -num).bit_length() - 1
    odd = num >> tz
    exp_lsb = tz - (den.bit_length() - 1)  # value = odd * 2^exp_lsb
    top = exp_lsb + odd.bit_length() - 1   # exponent of the leading bit
    if odd.bit_length() > 24:
        return False
    if top < -126:                          # subnormal range: lsb must be >= 2^-149
        return exp_lsb >= -149
    return exp_lsb >= top - 23


def nearest_ties_even(v: F, table):
    """Index of the table entry nearest to v (table sorted ascending); ties go to the even
    index; values beyond the last entry go to the last entry. Returns (index, robust_margin)
    where robust_margin is the distance from v to the nearest decision boundary."""
    best = None
    for i, t in enumerate(table):
        dist = abs(v - t)
        if best is None or dist < best[1] or (dist == best[1] and i % 2 == 0):
            best = (i, dist)
    i = best[0]
    # decision boundaries: midpoints between neighbours
    mids = [(table[k] + table[k + 1]) / 2 for k in range(len(table) - 1)]
    margin = min(abs(v - mp) for mp in mids)
    return i, margin


def round_f32(v: F) -> F:
    """Round an exact rational to the nearest binary32 (ties to even); overflow -> None."""
    if v == 0:
        return F(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if F(2) ** e > a:
        e -= 1
    q = F(2) ** (max(e, -126) - 23)       # quantum of that binade (subnormals below 2^-126)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * q
    if r > FLT_MAX:
        return None
    return sign * r
