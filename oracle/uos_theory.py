"""Data-free UOS objective -- TEST INFRASTRUCTURE (oracle side).

Restates the objective described on the Pith review page of "MXAttention:
Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
Attention" (referee summary of Sec. 4.1, Eqs. (21)-(23), Lemma 1, Theorem 1,
Table 6; Fig. 2 caption):

  Pi(v)  projection of v >= 0 onto the non-negative E2M1 grid
         {0, 0.5, 1, 1.5, 2, 3, 4, 6} (nearest point, saturating at 6)
  E(x)   = integral_0^x (v - Pi(v))^2 dv
  D(x)   = E(x) / x^3                       (scale-normalized error)
  J(q)   = E[D(X_q)], X_q the normalized block maximum under the ceiling rule
           with boundary q, i.e. X_q in (q/2, q] with log-domain density
           w(log2 x mod 1) (the periodized block-maximum law of Lemma 1).

E is evaluated exactly (piecewise cubic), J by Gauss-Legendre quadrature on
the pieces where the integrand is smooth.  Nothing here is used by the
product path.
"""
from __future__ import annotations

import math

import numpy as np

GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def projection(v: float) -> float:
    """Nearest non-negative E2M1 grid point (saturating at 6)."""
    if v >= GRID[-1]:
        return GRID[-1]
    return min(GRID, key=lambda g: abs(v - g))


def _breakpoints():
    """Grid points and the midpoints between neighbours: E's integrand is a
    single parabola (v - g)^2 between consecutive breakpoints."""
    pts = set(GRID)
    for a, b in zip(GRID[:-1], GRID[1:]):
        pts.add(0.5 * (a + b))
    return sorted(pts)


_BP = _breakpoints()


def E(x: float) -> float:
    """Exact integral of the squared projection error from 0 to x."""
    if x <= 0:
        return 0.0
    total = 0.0
    edges = [p for p in _BP if p < x] + [x]
    for lo, hi in zip(edges[:-1], edges[1:]):
        g = projection(0.5 * (lo + hi))  # the grid point that v in (lo, hi) rounds to
        total += ((hi - g) ** 3 - (lo - g) ** 3) / 3.0
    return total


def D(x: float) -> float:
    return E(x) / x ** 3


def Delta(q: float) -> float:
    """E(q) - 8 E(q/2): q^3 times D(q) - D(q/2), whose sign is the sign of J'(q)."""
    return E(q) - 8.0 * E(q / 2.0)


# Wrapped log-domain densities of the block maximum (period 1 in log2 units).
# The pages name log-uniform, first-harmonic, two-harmonic and concentrated
# densities without printing coefficients; these coefficients are our choice.
DENSITIES = {
    "log_uniform": lambda u: np.ones_like(u),
    "first_harmonic": lambda u: 1.0 + 0.6 * np.cos(2 * np.pi * (u - 0.3)),
    "two_harmonics": lambda u: 1.0 + 0.4 * np.cos(2 * np.pi * u) + 0.35 * np.sin(4 * np.pi * (u + 0.1)),
    "concentrated": lambda u: np.exp(4.0 * np.cos(2 * np.pi * (u - 0.65))),
}

_GL_X, _GL_W = np.polynomial.legendre.leggauss(24)


def J(q: float, w=DENSITIES["log_uniform"]) -> float:
    """E[D(X_q)] for X_q on (q/2, q] with density proportional to
    w(log2 x mod 1) / x (normalized over the interval)."""
    lo, hi = q / 2.0, q
    cuts = [lo] + [p for p in _BP if lo < p < hi] + [hi]
    # the density is smooth across log2 x = integer (w is periodic), but split there too
    for k in range(-2, 5):
        if lo < 2.0 ** k < hi:
            cuts.append(2.0 ** k)
    cuts = sorted(set(cuts))
    num = den = 0.0
    for a, b in zip(cuts[:-1], cuts[1:]):
        xs = 0.5 * (b - a) * _GL_X + 0.5 * (b + a)
        ws = 0.5 * (b - a) * _GL_W
        dens = w(np.mod(np.log2(xs), 1.0)) / xs
        dv = np.array([D(x) for x in xs])
        num += float(np.sum(ws * dens * dv))
        den += float(np.sum(ws * dens))
    return num / den


def argmin_J(w=DENSITIES["log_uniform"], lo=4.0, hi=8.0, coarse=0.01, tol=1e-9) -> float:
    """Minimize J over [lo, hi]: coarse grid, then golden-section refinement."""
    qs = np.arange(lo, hi + coarse / 2, coarse)
    vals = [J(q, w) for q in qs]
    i = int(np.argmin(vals))
    a, b = qs[max(i - 1, 0)], qs[min(i + 1, len(qs) - 1)]
    g = (math.sqrt(5) - 1) / 2
    c, d = b - g * (b - a), a + g * (b - a)
    fc, fd = J(c, w), J(d, w)
    while b - a > tol:
        if fc < fd:
            b, d, fd = d, c, fc
            c = b - g * (b - a)
            fc = J(c, w)
        else:
            a, c, fc = c, d, fd
            d = a + g * (b - a)
            fd = J(d, w)
    return 0.5 * (a + b)


def root_of_Delta(lo=7.0, hi=8.0, tol=1e-14) -> float:
    """Bisection for the sign change of Delta on [lo, hi]."""
    flo = Delta(lo)
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        fm = Delta(mid)
        if (fm < 0) == (flo < 0):
            lo, flo = mid, fm
        else:
            hi = mid
        if hi - lo < tol:
            break
    return 0.5 * (lo + hi)
