"""Exact IEEE rounding in rational arithmetic, for the oracle's pins.

Independent of numpy's float32/float16 casts: values are Fractions and every
rounding is written out (round to nearest, ties to even, with the format's
precision and exponent range).
"""
from fractions import Fraction


def round_binary(x: Fraction, p: int, emin: int, emax: int):
    """Exact IEEE round-to-nearest-even of x to p significand bits; None = overflow."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - p + 1)
    m = a / quantum
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    r = fl * quantum
    if r >= Fraction(2) ** (emax + 1):
        return None
    return sign * r


def f32(x):
    return round_binary(x, 24, -126, 127)


def f16(x):
    return round_binary(x, 11, -14, 15)


def nearest_q(w: Fraction, s: Fraction) -> int:
    """Brute force: the q in [-7, 7] closest to w/s, ties to the even q."""
    best = None
    for q in range(-7, 8):
        d = abs(w - q * s)
        if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
            best = (d, q)
    return best[1]
