"""Exact-arithmetic helpers for brute-force pins of the oracle (tests only).

These use Python's ``fractions.Fraction`` so that every rounding decision can
be checked against the exact rational value, independently of numpy.
"""

from fractions import Fraction

import numpy as np


def f32_rne(x: Fraction) -> float:
    """Exact round-to-nearest-even of a rational to IEEE binary32 (finite range)."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    a = abs(x)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    q_exp = max(e, -126) - 23                 # quantum exponent (subnormals: 2^-149)
    quantum = Fraction(2) ** q_exp
    m = a / quantum
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    val = float(Fraction(fl) * quantum)       # exactly representable
    out = np.float32(sign * val)
    assert Fraction(float(out)) == sign * Fraction(fl) * quantum
    return float(out)


def round_half_even(x: Fraction) -> int:
    fl = x.numerator // x.denominator
    rem = x - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return fl


def nearest_level_exact(n: float, levels) -> int:
    """argmin_i |n - v_i| over exact rationals; ties -> lower index."""
    fn = Fraction(float(n))
    best, best_d = None, None
    for i, v in enumerate(levels):
        d = abs(fn - Fraction(float(v)))
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


def round_binary(x: Fraction, p: int, emin: int) -> Fraction:
    """Exact round-to-nearest-even of a rational to a binary format with p
    significant bits and smallest normal exponent emin (gradual underflow below
    it, no overflow handling).  Returns the rounded value as a Fraction; a
    result of zero carries no sign, so callers decide the sign of zero."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, emin) - (p - 1))
    m = a / quantum
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * Fraction(fl) * quantum


def bf16_bits_exact(x: Fraction, negative_zero: bool = False) -> int:
    """bf16 round-to-nearest-even of a rational (8 significant bits, the fp32
    exponent range), as the 16-bit pattern.  Built from the value, not from an
    fp32 bit pattern: sign, biased exponent and stored fraction are derived
    from the rounded rational.  `negative_zero` gives the sign of a zero."""
    v = round_binary(x, 8, -126)
    if v == 0:   # an exact zero takes the given sign; a value that underflows keeps its own
        return 0x8000 if (negative_zero if x == 0 else x < 0) else 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    if e < -126:                                  # subnormal: value = f * 2^-133
        f = a / Fraction(2) ** -133
        assert f.denominator == 1 and f < 128
        return sign | int(f)
    assert e <= 127, "bf16 overflow"
    frac = a / Fraction(2) ** e - 1               # in [0, 1), a multiple of 2^-7
    f = frac * 128
    assert f.denominator == 1
    return sign | ((e + 127) << 7) | int(f)


def f32_from_fraction(v: Fraction, negative_zero: bool = False) -> np.float32:
    """An exactly representable rational as np.float32 (sign of zero given)."""
    if v == 0:
        return np.float32(-0.0) if negative_zero else np.float32(0.0)
    out = np.float32(float(v))
    assert Fraction(float(out)) == v
    return out
