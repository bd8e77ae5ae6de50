"""Exact evaluation of the time bucket floor(ln(x)/0.301) with decimal arithmetic.

Independent of the oracle and of the CUDA library: it derives the bucket edges
e^(0.301 b) at 60 significant digits and counts the edges at or below x.
Used by the tests only, as the mathematical pin for both sides.
"""
from __future__ import annotations

import decimal
from functools import lru_cache

_CTX = decimal.Context(prec=60)


@lru_cache(maxsize=None)
def edges(num_buckets: int = 128):
    """E_b = e^(0.301*b) for b = 0..num_buckets-1 as Decimals."""
    step = _CTX.multiply(decimal.Decimal("0.301"), 1)
    return tuple(_CTX.exp(_CTX.multiply(step, b)) for b in range(num_buckets))


@lru_cache(maxsize=None)
def integer_thresholds(num_buckets: int = 128):
    """thr_b = smallest integer x with x >= E_b, i.e. ln(x) >= 0.301 b."""
    out = []
    for e in edges(num_buckets):
        c = int(e.to_integral_value(rounding=decimal.ROUND_CEILING))
        out.append(c)
    return tuple(out)


def min_edge_gap(num_buckets: int = 128) -> decimal.Decimal:
    """Smallest distance of an edge E_b (b >= 1) to an integer."""
    gaps = []
    for e in edges(num_buckets)[1:]:
        frac = e - e.to_integral_value(rounding=decimal.ROUND_FLOOR)
        gaps.append(min(frac, 1 - frac))
    return min(gaps)


def bucket(dt: int, num_buckets: int = 128) -> int:
    x = abs(int(dt)) + 1
    thr = integer_thresholds(num_buckets)
    b = 0
    for i in range(1, num_buckets):
        if thr[i] <= x:
            b = i
    return b


def bucket_direct(dt: int, num_buckets: int = 128) -> int:
    """floor(ln(|dt|+1)/0.301) evaluated directly in 60-digit decimal."""
    x = decimal.Decimal(abs(int(dt)) + 1)
    val = _CTX.divide(_CTX.ln(x), decimal.Decimal("0.301"))
    b = int(val.to_integral_value(rounding=decimal.ROUND_FLOOR))
    return max(0, min(num_buckets - 1, b))
