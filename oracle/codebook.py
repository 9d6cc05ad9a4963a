"""Lloyd-Max scalar quantizer for the standard normal — oracle (test only).

[TQAI §The Paper]: after the random rotation each coordinate of a unit vector
is modelled as N(0, 1/d), so the optimal (Lloyd-Max) scalar quantizer can be
computed once, offline, without data. [ADAPTQ §How it works, item 2]: the
rotated vectors are scalar-quantized with Max-Lloyd codebooks.

Everything here is in N(0,1) units; the N(0,1/d) codebook is these values
divided by sqrt(d).

Lloyd-Max conditions for N = 2^b levels (Max 1960; Lloyd 1982):
  centroid   c_j = E[X | t_j <= X < t_{j+1}]   (t_0 = -inf, t_N = +inf)
  midpoint   t_j = (c_{j-1} + c_j) / 2          j = 1..N-1
The density is symmetric, so the solution is symmetric and the middle
threshold is 0; the iteration runs on the positive half-line.
"""
from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def pdf(x: float) -> float:
    """Standard normal density; 0 at +-inf."""
    if math.isinf(x):
        return 0.0
    return _INV_SQRT_2PI * math.exp(-0.5 * x * x)


def upper_tail(x: float) -> float:
    """P(X > x) for X ~ N(0,1), via erfc (accurate in the upper tail)."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / _SQRT2)


def cell_mass(a: float, b: float) -> float:
    """P(a < X < b) for 0 <= a < b (positive half-line cells)."""
    return upper_tail(a) - upper_tail(b)


def cell_centroid(a: float, b: float) -> float:
    """E[X | a < X < b] = (phi(a) - phi(b)) / P(a < X < b)."""
    return (pdf(a) - pdf(b)) / cell_mass(a, b)


def lloyd_max_normal(bits: int, tol: float = 1e-14, max_iter: int = 200000):
    """Solve the Lloyd-Max fixed point for N(0,1) with 2^bits levels.

    Returns (centroids[N], thresholds[N-1]) as float64 arrays, ascending.
    Start: centroids at equal-probability quantiles of the half-normal.
    Iterate midpoint and centroid updates until the largest change < tol.
    """
    if not 1 <= bits <= 8:
        raise ValueError("bits must be in 1..8")
    n_levels = 1 << bits
    half = n_levels // 2
    inv = NormalDist().inv_cdf
    # positive half: cells k = 0..half-1, each with mass 0.5/half initially
    c = [inv(0.5 + 0.5 * (k + 0.5) / half) for k in range(half)]
    for _ in range(max_iter):
        t = [0.0] + [0.5 * (c[k - 1] + c[k]) for k in range(1, half)] + [math.inf]
        new_c = [cell_centroid(t[k], t[k + 1]) for k in range(half)]
        delta = max(abs(x - y) for x, y in zip(new_c, c))
        c = new_c
        if delta < tol:
            break
    else:
        raise RuntimeError("Lloyd-Max iteration did not converge")
    t_pos = [0.5 * (c[k - 1] + c[k]) for k in range(1, half)]
    centroids = np.array([-x for x in reversed(c)] + c, dtype=np.float64)
    thresholds = np.array([-x for x in reversed(t_pos)] + [0.0] + t_pos,
                          dtype=np.float64)
    return centroids, thresholds


def quantizer_mse(centroids: np.ndarray, thresholds: np.ndarray) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1), summed cell by cell in closed form.

    On a cell (a, b) with level c:
      integral (x - c)^2 phi(x) dx = P + a*phi(a) - b*phi(b)
                                     - 2c*(phi(a) - phi(b)) + c^2 * P
    with P = P(a < X < b); a*phi(a) is 0 at a = -inf.
    """
    edges = [-math.inf] + [float(x) for x in thresholds] + [math.inf]
    total = 0.0
    for j, c in enumerate(centroids):
        a, b = edges[j], edges[j + 1]
        p = upper_tail(a) - upper_tail(b)
        apa = 0.0 if math.isinf(a) else a * pdf(a)
        bpb = 0.0 if math.isinf(b) else b * pdf(b)
        total += p + apa - bpb - 2.0 * c * (pdf(a) - pdf(b)) + c * c * p
    return total


def codebook(bits: int):
    """(centroids, thresholds, mse) in N(0,1) units."""
    c, t = lloyd_max_normal(bits)
    return c, t, quantizer_mse(c, t)
