"""Lloyd-Max 16-level scalar quantiser for the standard normal distribution (float64).

TEST INFRASTRUCTURE ONLY.  This module belongs to the float64 CPU oracle.  Only the
test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it; the CUDA library computes its own copy of the table independently.

Method (the compact tier of "Context beyond VRAM", section "What I built": older
history is held in a compact form the GPU reads directly; the 16-level table for
N(0,1) is the one the hybrid-tier workload names): a Lloyd-Max quantiser satisfies
two conditions at once --
  * every decision boundary is the midpoint of its two neighbouring levels, and
  * every level is the conditional mean of N(0,1) over its cell,
      c_j = (phi(a) - phi(b)) / (Phi(b) - Phi(a))   for the cell (a, b).
Lloyd's iteration alternates the two conditions until the levels stop moving.
The fixed point for a log-concave density is unique, so the starting point only
affects the iteration count.  The float64 levels are then made exactly odd-symmetric
and rounded to IEEE binary16 (round-to-nearest-even): that binary16 table is the
canonical centroid table of the compact tier.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np

LEVELS = 16

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _upper_tail(x: float) -> float:
    """P(X > x) for X ~ N(0,1), accurate in the upper tail."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / _SQRT2)


def _pdf(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return _INV_SQRT_2PI * math.exp(-0.5 * x * x)


def cell_mass(a: float, b: float) -> float:
    """P(a < X < b) for X ~ N(0,1), using whichever tail keeps the difference accurate."""
    if a >= 0.0:
        return _upper_tail(a) - _upper_tail(b)
    if b <= 0.0:
        return _upper_tail(-b) - _upper_tail(-a)
    return 1.0 - _upper_tail(-a) - _upper_tail(b)


def conditional_mean(a: float, b: float) -> float:
    """E[X | a < X < b] for X ~ N(0,1): (phi(a) - phi(b)) / P(a < X < b)."""
    return (_pdf(a) - _pdf(b)) / cell_mass(a, b)


def boundaries(levels: np.ndarray) -> np.ndarray:
    """Decision boundaries of a sorted level set: the midpoints of neighbours."""
    levels = np.asarray(levels, dtype=np.float64)
    return (levels[:-1] + levels[1:]) / 2.0


def lloyd_step(levels: np.ndarray) -> np.ndarray:
    """One Lloyd iteration: midpoint boundaries, then the conditional mean of each cell."""
    edges = [-math.inf, *boundaries(levels).tolist(), math.inf]
    return np.array([conditional_mean(edges[j], edges[j + 1]) for j in range(len(levels))])


@lru_cache(maxsize=None)
def lloyd_max_normal_f64(levels: int = LEVELS, tol: float = 1e-15, max_iter: int = 100_000) -> tuple:
    """Float64 Lloyd-Max levels for N(0,1), ascending, made exactly odd-symmetric.

    Starts from uniform levels on [-2.7, 2.7] and iterates until no level moves by
    more than ``tol``.  Returns a tuple (hashable for the cache)."""
    c = np.linspace(-2.7, 2.7, levels)
    for _ in range(max_iter):
        c_next = lloyd_step(c)
        moved = float(np.max(np.abs(c_next - c)))
        c = c_next
        if moved <= tol:
            break
    else:  # pragma: no cover - convergence is checked by the tests
        raise RuntimeError("Lloyd iteration did not converge")
    c = (c - c[::-1]) / 2.0  # exact odd symmetry: c[L-1-j] = -c[j]
    return tuple(float(x) for x in c)


def centroids_f16_bits() -> np.ndarray:
    """The canonical table as IEEE binary16 bit patterns (uint16[16], ascending values)."""
    c = np.array(lloyd_max_normal_f64(), dtype=np.float64)
    return c.astype(np.float16).view(np.uint16)


def centroids_f16() -> np.ndarray:
    """The canonical table as float64 values of the binary16 levels (exact)."""
    return centroids_f16_bits().view(np.float16).astype(np.float64)


def quantiser_mse(levels: np.ndarray) -> float:
    """Mean squared error E[(X - Q(X))^2] of a nearest-level quantiser for N(0,1).

    Per cell (a, b) with level c: E[X^2 1] - 2c E[X 1] + c^2 P, where
    E[X^2 1{a<X<b}] = P + a phi(a) - b phi(b) and E[X 1{a<X<b}] = phi(a) - phi(b)."""
    levels = np.asarray(levels, dtype=np.float64)
    edges = [-math.inf, *boundaries(levels).tolist(), math.inf]
    total = 0.0
    for j, c in enumerate(levels):
        a, b = edges[j], edges[j + 1]
        p = cell_mass(a, b)
        a_phi = 0.0 if math.isinf(a) else a * _pdf(a)
        b_phi = 0.0 if math.isinf(b) else b * _pdf(b)
        second = p + a_phi - b_phi
        first = _pdf(a) - _pdf(b)
        total += second - 2.0 * c * first + c * c * p
    return total
