"""Exact rational references used to pin the oracle (independent of it).

``rne_bf16`` rounds an exact rational to bf16 by the definition of round-to-nearest-even: it
looks up the two neighbouring representable bf16 values in the sorted table of all finite
positive bf16 numbers (decoded with a numpy bit view, not with the oracle's codec), picks the
nearer one and, on a tie, the one whose bit pattern is even.  No quantum/exponent arithmetic is
shared with the oracle's fp64 -> bf16 routine.
"""
from __future__ import annotations

import bisect
from fractions import Fraction

import numpy as np

_POS_BITS = np.arange(0x0000, 0x7F80, dtype=np.uint32)          # +0 .. largest finite
_POS_VALS = (_POS_BITS << 16).astype(np.uint32).view(np.float32).astype(np.float64)
_POS_FRAC = [Fraction(float(v)) for v in _POS_VALS]
_OVERFLOW = Fraction(2) ** 128   # the value the next pattern (0x7F80) would have if it were finite


def rne_bf16(q: Fraction) -> int:
    """Exact rational -> bf16 bit pattern, round to nearest, ties to even."""
    q = Fraction(q)
    sign = 0x8000 if q < 0 else 0
    a = abs(q)
    if a == 0:
        return 0  # an exact zero sum is +0 under round-to-nearest
    i = bisect.bisect_left(_POS_FRAC, a)
    if i < len(_POS_FRAC) and _POS_FRAC[i] == a:
        return sign | int(_POS_BITS[i])
    lo_bits = int(_POS_BITS[i - 1])
    lo = _POS_FRAC[i - 1]
    if i < len(_POS_FRAC):
        hi_bits, hi = int(_POS_BITS[i]), _POS_FRAC[i]
    else:
        hi_bits, hi = 0x7F80, _OVERFLOW
    dlo, dhi = a - lo, hi - a
    if dlo < dhi:
        bits = lo_bits
    elif dhi < dlo:
        bits = hi_bits
    else:
        bits = lo_bits if lo_bits % 2 == 0 else hi_bits
    return sign | bits


def bf16_bits_to_fraction(bits: int) -> Fraction:
    """Exact value of a finite bf16 pattern, via a numpy float32 view."""
    v = np.array([(bits & 0xFFFF) << 16], dtype=np.uint32).view(np.float32)[0]
    return Fraction(float(v))


def exact_gemm(A, B):
    """Exact rational C = A . B^T for small float arrays (lists of Fractions)."""
    A = [[Fraction(float(x)) for x in row] for row in np.asarray(A)]
    B = [[Fraction(float(x)) for x in row] for row in np.asarray(B)]
    return [[sum((a * b for a, b in zip(ra, rb)), Fraction(0)) for rb in B] for ra in A]
