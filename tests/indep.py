"""Independent checks used to pin the oracle (numpy + exact rationals).

Nothing here is imported by the oracle or by the library.  The nearest-point
search below is a second, differently written brute force: binary64 distances
from numpy select a short list, and Python ``fractions.Fraction`` decides it
exactly, ties going to the smallest index.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def exact_dist2(u, point_num, den):
    """|u - point_num/den|^2 exactly (u: fp32 values, point_num: integers)."""
    s = Fraction(0)
    for ui, pi in zip(u, point_num):
        d = Fraction(float(ui)) - Fraction(int(pi), den)
        s += d * d
    return s


def nearest_exact(u, cand_num, den):
    """Smallest index among the exact minimisers of |u - cand/den|^2.

    cand_num: int array [n, 8] of numerators."""
    u = np.asarray(u, dtype=np.float32)
    C = cand_num.astype(np.float64) / den
    d = ((u.astype(np.float64)[None, :] - C) ** 2).sum(1)
    dmin = d.min()
    short = np.nonzero(d <= dmin * (1 + 1e-9) + 1e-300)[0]
    best, bestd = None, None
    for c in short:
        e = exact_dist2(u, cand_num[c], den)
        if bestd is None or e < bestd:
            best, bestd = int(c), e
    return best


def stage1_exact(u, cb):
    return nearest_exact(u, cb.astype(np.int64), 2)


def stage2_exact(u, cb, i1, bpw):
    m = 4 if bpw == 3 else 8
    n = 256 if bpw == 3 else len(cb)
    num = (m // 2) * cb[i1].astype(np.int64)[None, :] + cb[:n].astype(np.int64)
    return nearest_exact(u, num, m)


def sylvester(n):
    """Sylvester-Hadamard matrix, H[i][j] = (-1)^popcount(i & j)."""
    i = np.arange(n)
    pc = np.zeros((n, n), dtype=np.int64)
    a = i[:, None] & i[None, :]
    while np.any(a):
        pc += a & 1
        a = a >> 1
    return np.where(pc % 2 == 0, 1, -1).astype(np.int64)


def splitmix64_reference_outputs():
    """First outputs of SplitMix64 seeded with 0 (published known-answer values)."""
    return [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def theta_e8(m):
    """Number of E8 vectors of squared norm 2m: 240 sigma_3(m) (m >= 1), 1 for m = 0."""
    if m == 0:
        return 1
    return 240 * sum(d ** 3 for d in range(1, m + 1) if m % d == 0)
