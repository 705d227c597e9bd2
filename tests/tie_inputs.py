"""Weights whose MinMax groups put many elements exactly half-way between two
grid points, so that the rounding rule (half to even) decides their codes.

Every group has min = -z0 * s and max = (Q - z0) * s (or the same shifted by
half a step, so that the zero point itself is a tie), with s = c * 2^-e an
exact fp16 number: the range is exactly Q * s, the scale is exactly s, and the
other elements are (j + 1/2) * s, whose quotient by the scale is exactly
j + 1/2.  All values are exact in bf16.  The expected codes and zeros follow
from exact rational arithmetic and Python's round() (half to even), without
the oracle.
"""
from fractions import Fraction

import numpy as np


def tie_weight(n: int, k: int, bits: int, seed: int):
    """Returns (w float32 [n, k], codes int64 [n, k], zero int64 [n, k/g],
    scale float64 [n, k/g]) for groups of 128 (bits 4) or 64 (bits 2)."""
    Q = (1 << bits) - 1
    group = 128 if bits == 4 else 64
    rng = np.random.default_rng(seed)
    w = np.empty((n, k), np.float64)
    codes = np.empty((n, k), np.int64)
    ng = k // group
    zeros = np.empty((n, ng), np.int64)
    scales = np.empty((n, ng), np.float64)
    for i in range(n):
        for g in range(ng):
            c = int(rng.choice([1, 3, 5, 7]))
            e = int(rng.integers(6, 11))
            s = Fraction(c, 2 ** e)
            z0 = int(rng.integers(0, Q + 1))
            half_zero = bool(rng.integers(0, 2)) and z0 < Q
            lo = -(Fraction(z0) + (Fraction(1, 2) if half_zero else 0))   # min / s
            hi = lo + Q                                                 # max / s
            # interior points: half-integers j + 1/2 within [lo, hi]
            cand = [Fraction(2 * j + 1, 2) for j in range(-Q - 1, Q + 1)]
            cand = [t for t in cand if lo <= t <= hi]
            t = [lo, hi] + [cand[int(x)] for x in rng.integers(0, len(cand), group - 2)]
            t = [t[int(x)] for x in rng.permutation(group)]
            vals = [tt * s for tt in t]
            w[i, g * group:(g + 1) * group] = [float(v) for v in vals]
            z = round(-lo)                                               # half to even
            zeros[i, g] = z
            scales[i, g] = float(s)
            codes[i, g * group:(g + 1) * group] = [min(max(round(tt) + z, 0), Q) for tt in t]
    return w.astype(np.float32), codes, zeros, scales
