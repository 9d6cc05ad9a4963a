"""Randomized Hadamard rotation — oracle (test only).

[ADAPTQ §How it works, item 1]: y = (1/sqrt d) · H · D · x, with H a Hadamard
matrix applied by a fast Walsh-Hadamard transform and D a random diagonal of
+-1 entries; the rotation spreads outlier energy over all coordinates.
[TQAI §The Paper]: rotate, then quantize coordinate by coordinate.

The oracle forms H densely from its definition and multiplies; no FWHT.
  H[i][j] = (-1)^popcount(i & j)  (Sylvester order, entries +-1, unnormalized)
  R       = H · diag(D) / sqrt(d)  (orthonormal, since H·H = d·I and D·D = I)
  R^T     = diag(D) · H / sqrt(d)

The pages name no generator for D. The library's definition: SplitMix64
(Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014) with its state set to the seed; D_i = -1 iff bit 63 of the i-th
64-bit output (i = 0, 1, ...) is set.
"""
from __future__ import annotations

import numpy as np

_MASK64 = (1 << 64) - 1
_GOLDEN_GAMMA = 0x9E3779B97F4A7C15


def splitmix64(seed: int, n: int) -> list:
    """First n outputs of SplitMix64 whose state starts at `seed`."""
    state = seed & _MASK64
    out = []
    for _ in range(n):
        state = (state + _GOLDEN_GAMMA) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def sign_vector(seed: int, d: int) -> np.ndarray:
    """D as float64 +-1 entries: -1 where bit 63 of output i is set."""
    return np.array([-1.0 if (v >> 63) & 1 else 1.0 for v in splitmix64(seed, d)],
                    dtype=np.float64)


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order d (a power of two), float64 +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.empty((d, d), dtype=np.float64)
    for i in range(d):
        for j in range(d):
            h[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return h


def rotate(x: np.ndarray, seed: int) -> np.ndarray:
    """y = (1/sqrt d) · H · (D ⊙ x) for each row of x ([..., d])."""
    d = x.shape[-1]
    return (x * sign_vector(seed, d)) @ hadamard(d).T / np.sqrt(d)


def unrotate(y: np.ndarray, seed: int) -> np.ndarray:
    """x = R^T y = D ⊙ (H · y) / sqrt(d) for each row of y ([..., d])."""
    d = y.shape[-1]
    return sign_vector(seed, d) * (y @ hadamard(d).T) / np.sqrt(d)
