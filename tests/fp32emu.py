"""Exactly rounded fp32 arithmetic for host tests: an operation is evaluated in rational
arithmetic and rounded once to fp32, to nearest (ties to even), up or down."""
from fractions import Fraction as Fr

import numpy as np


def round_f32(x, mode):
    """x (a Fraction) rounded to fp32: 'rn', 'ru' or 'rd'. Returns a Python float (finite range)."""
    g = np.float32(float(x))
    lo = hi = g
    while Fr(float(lo)) > x:
        lo = np.nextafter(lo, np.float32(-np.inf), dtype=np.float32)
    while Fr(float(hi)) < x:
        hi = np.nextafter(hi, np.float32(np.inf), dtype=np.float32)
    if Fr(float(lo)) < x:  # lo is the largest value below x; hi the smallest above
        hi = np.nextafter(lo, np.float32(np.inf), dtype=np.float32)
    if Fr(float(hi)) > x:
        lo = np.nextafter(hi, np.float32(-np.inf), dtype=np.float32)
    if lo == hi or Fr(float(lo)) == x:
        return float(lo)
    if mode == "ru":
        return float(hi)
    if mode == "rd":
        return float(lo)
    dl, dh = x - Fr(float(lo)), Fr(float(hi)) - x
    if dl != dh:
        return float(lo if dl < dh else hi)
    return float(lo if (np.float32(lo).view(np.uint32) & 1) == 0 else hi)


def fma_f32(a, b, c, mode="rn"):
    return round_f32(Fr(a) * Fr(b) + Fr(c), mode)
