"""Exact model of IEEE-754 binary32 round-to-nearest-even arithmetic.

Each operation is carried out on exact rationals (``fractions.Fraction``) and
then rounded once to the nearest binary32 value, ties to even -- the
definition of a correctly rounded IEEE operation.  The tests use it to
re-derive the fp32 neighbor predicate from its written definition, without
sharing any arithmetic with the C oracle or the CUDA kernels.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

_EMIN = -126
_MANT = 23


def round_f32(q: Fraction, neg_zero: bool = False) -> float:
    """Nearest binary32 value to the exact rational q (ties to even)."""
    if q == 0:
        return -0.0 if neg_zero else 0.0
    sign = -1.0 if q < 0 else 1.0
    a = -q if q < 0 else q
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    if e < _EMIN:
        scale = Fraction(2) ** (_EMIN - _MANT)
    else:
        scale = Fraction(2) ** (e - _MANT)
    m = a / scale
    mi = round(m)  # Fraction.__round__ rounds half to even
    if e > 127 or (mi * scale) >= Fraction(2) ** 128:
        return sign * math.inf
    v = float(mi * scale)  # exact in float64
    out = float(np.float32(v))
    assert out == v, "rounding model produced a non-binary32 value"
    return sign * out


def F(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def add(a, b) -> float:
    return round_f32(F(a) + F(b))


def sub(a, b) -> float:
    return round_f32(F(a) - F(b))


def mul(a, b) -> float:
    return round_f32(F(a) * F(b))


def div(a, b) -> float:
    return round_f32(F(a) / F(b))


def floor_(a) -> float:
    return float(math.floor(F(a)))


def rint_(a) -> float:
    return float(round(F(a)))  # half to even


def wrap(x, L) -> float:
    """x - L*floor(x/L), one correction into [0, L), else 0."""
    t = floor_(div(x, L))
    w = sub(x, mul(L, t))
    if w < 0:
        w = add(w, L)
    if w >= float(np.float32(L)):
        w = sub(w, L)
    if not (0 <= w < float(np.float32(L))):
        w = 0.0
    return w


def min_image(d, L) -> float:
    return sub(d, mul(L, rint_(div(d, L))))


def r2(a, b, box) -> float:
    """((dx*dx + dy*dy) + dz*dz) with d = min_image(b - a)."""
    d = [min_image(sub(b[k], a[k]), box[k]) for k in range(3)]
    s = add(mul(d[0], d[0]), mul(d[1], d[1]))
    return add(s, mul(d[2], d[2]))
