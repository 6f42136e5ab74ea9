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
