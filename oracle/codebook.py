"""Lloyd-Max scalar quantizer for a Gaussian source (oracle side; test infrastructure only).

The rotated 4-bit format stores, per coordinate, an index into a 16-entry
codebook fitted to N(0, sigma^2) with sigma^2 = 1/D: after a random-sign
Walsh-Hadamard rotation and division by the vector norm, each coordinate of a
unit vector is close to N(0, 1/D).  The codebook is the minimum-MSE one, found
by Lloyd's iteration (Lloyd 1957 / Max 1960):

    thresholds  t_i = (c_i + c_{i+1}) / 2
    centroids   c_i = E[X | t_{i-1} < X < t_i]
                    = sigma * (phi(a) - phi(b)) / (Phi(b) - Phi(a)),
                      a = t_{i-1}/sigma, b = t_i/sigma

iterated in fp64 until the centroids move by less than 1e-13 sigma.  The density
is symmetric, so the optimum is too; each iterate is symmetrized
(c <- (c - reverse(c)) / 2) so that rounding cannot break the symmetry.
The library stores the codebook as float16 (the precision of the cache's other
per-vector parameters); ``lloyd_max_f16`` gives that rounding.
"""
from __future__ import annotations

import math

import numpy as np


def _phi(z: float) -> float:
    return math.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi) if math.isfinite(z) else 0.0


def _Phi(z: float) -> float:
    if z == math.inf:
        return 1.0
    if z == -math.inf:
        return 0.0
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


def lloyd_max_gaussian(levels: int = 16, sigma: float = 1.0, tol: float = 1e-13,
                       max_iter: int = 200000):
    """Return (centroids, thresholds, iterations) in fp64; centroids increasing."""
    c = np.linspace(-2.0, 2.0, levels)
    it = 0
    for it in range(1, max_iter + 1):
        t = np.concatenate([[-math.inf], 0.5 * (c[:-1] + c[1:]), [math.inf]])
        new = np.empty_like(c)
        for i in range(levels):
            a, b = t[i], t[i + 1]
            mass = _Phi(b) - _Phi(a)
            new[i] = (_phi(a) - _phi(b)) / mass
        new = 0.5 * (new - new[::-1])
        delta = float(np.max(np.abs(new - c)))
        c = new
        if delta < tol:
            break
    t = 0.5 * (c[:-1] + c[1:])
    return c * sigma, t * sigma, it


def lloyd_max_f16(levels: int = 16, sigma: float = 1.0) -> np.ndarray:
    """The codebook as the library stores it: float16, round-to-nearest-even."""
    c, _, _ = lloyd_max_gaussian(levels, sigma)
    return c.astype(np.float16)


def gaussian_mse(centroids: np.ndarray, sigma: float = 1.0) -> float:
    """Mean squared error of nearest-centroid quantization of N(0, sigma^2) (closed form)."""
    c = np.asarray(centroids, dtype=np.float64) / sigma
    t = np.concatenate([[-math.inf], 0.5 * (c[:-1] + c[1:]), [math.inf]])
    total = 0.0
    for i in range(len(c)):
        a, b = t[i], t[i + 1]
        m0 = _Phi(b) - _Phi(a)                      # P(a < X < b)
        m1 = _phi(a) - _phi(b)                      # E[X 1{a<X<b}]
        # E[X^2 1{a<X<b}] = m0 + a phi(a) - b phi(b)   (with z phi(z) -> 0 at +-inf)
        za = a * _phi(a) if math.isfinite(a) else 0.0
        zb = b * _phi(b) if math.isfinite(b) else 0.0
        m2 = m0 + za - zb
        total += m2 - 2.0 * c[i] * m1 + c[i] * c[i] * m0
    return total * sigma * sigma
