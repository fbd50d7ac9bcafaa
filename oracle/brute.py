"""Pure-Python brute force for tiny cases -- TEST INFRASTRUCTURE ONLY.

Independent second readings used to pin :mod:`oracle.wushkv_oracle`:
nearest-level search over every level, softmax attention written with
explicit loops, and fp16 rounding done with exact rational arithmetic.
Nothing here is vectorised and nothing is shared with the oracle's code.
"""
from __future__ import annotations

import math
from fractions import Fraction


def fp16_round_exact(x: float) -> float:
    """Round a finite float to the nearest fp16 value, ties to even, using
    exact rationals (IEEE 754 binary16: 10 fraction bits, emin = -14,
    subnormal step 2^-24, max finite 65504)."""
    if x == 0.0 or math.isnan(x):
        return x
    sign = -1.0 if x < 0 else 1.0
    a = Fraction(abs(x))
    if a >= Fraction(65520):            # rounds to infinity
        return sign * math.inf
    e = math.floor(math.log2(abs(x)))
    # guard against log2 rounding at exact powers of two
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -14)
    ulp = Fraction(2) ** (e - 10)
    q, r = divmod(a, ulp)
    half = ulp / 2
    if r > half or (r == half and q % 2 == 1):
        q += 1
    return sign * float(q * ulp)


def nearest_level(x: float, levels: list[float]) -> list[int]:
    """Indices of all levels at minimal distance from x."""
    best = min(abs(x - v) for v in levels)
    return [i for i, v in enumerate(levels) if abs(x - v) == best]


def attention_loops(q: list[float], K: list[list[float]], V: list[list[float]],
                    scale: float) -> list[float]:
    """softmax(scale * q.K^T) V with explicit loops (no max subtraction;
    inputs are kept small by the callers)."""
    n, d = len(K), len(q)
    w = []
    for t in range(n):
        s = 0.0
        for j in range(d):
            s += q[j] * K[t][j]
        w.append(math.exp(scale * s))
    z = sum(w)
    out = []
    for j in range(len(V[0])):
        acc = 0.0
        for t in range(n):
            acc += w[t] * V[t][j]
        out.append(acc / z)
    return out


def matvec(M: list[list[float]], x: list[float]) -> list[float]:
    return [sum(M[i][j] * x[j] for j in range(len(x))) for i in range(len(M))]
