"""Polar Express coefficient schedule by linear programming (fp64 CPU oracle).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: it shares no code
with the CUDA library and imports nothing from it.

The source pages name a "production Polar Express" schedule for the
Newton-Schulz step but print no coefficients.  The construction followed
here is the greedy minimax one of Amsel, Persson, Musco and Gower, "The
Polar Express: Optimal Matrix Sign Methods and Their Application to the
Muon Algorithm" (2025):

* after t steps every singular value of the normalized input lies in an
  interval [lo_t, hi_t]; the first is [lower, 1];
* step t applies the odd quintic p(x) = a x + b x^3 + c x^5 minimizing
  max |1 - p(x)| over [lo_t, hi_t];
* the next interval is the image of [lo_t, hi_t] under the polynomial
  applied.

Readings (the same ones the library states): a safety factor s >= 1 applies
p(x / s) instead of p; an interval narrower than 1e-3 takes the quintic with
p(1) = 1, p'(1) = p''(1) = 0, i.e. (15/8, -5/4, 3/8).

Where the library runs a Remez exchange, this oracle solves the discretized
minimax problem as a linear program over a dense Chebyshev grid (variables
a, b, c, E; minimize E subject to |1 - p(x_j)| <= E at every grid point),
and takes the interval's image by dense evaluation refined at the roots of
p' -- a different method for the same definition.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np

__all__ = ["minimax_quintic_lp", "polar_express_lp", "quintic_image", "FIXED_POINT_QUINTIC"]

FIXED_POINT_QUINTIC = (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)


def _p(coef, x):
    a, b, c = coef
    return a * x + b * x ** 3 + c * x ** 5


def minimax_quintic_lp(lo: float, hi: float, points: int = 4001) -> Tuple[Tuple[float, float, float], float]:
    """Odd quintic minimizing max |1 - p| over a Chebyshev grid of [lo, hi], and that maximum."""
    from scipy.optimize import linprog

    k = np.arange(points)
    x = 0.5 * (lo + hi) - 0.5 * (hi - lo) * np.cos(np.pi * k / (points - 1))
    # Solved in the variable t = x / hi (coefficients a hi, b hi^3, c hi^5):
    # the same problem, but with columns t, t^3, t^5 of comparable size on any
    # interval, which keeps the solver's tolerance small next to E.
    t = x / hi
    V = np.stack([t, t ** 3, t ** 5], axis=1)
    ones = np.ones((points, 1))
    # 1 - p(x) <= E  ->  -V z - E <= -1 ;   p(x) - 1 <= E  ->  V z - E <= 1
    A_ub = np.vstack([np.hstack([-V, -ones]), np.hstack([V, -ones])])
    b_ub = np.concatenate([-np.ones(points), np.ones(points)])
    res = linprog(c=[0.0, 0.0, 0.0, 1.0], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
    if not res.success:
        raise RuntimeError(f"linear program failed: {res.message}")
    a, b, c, E = res.x
    return (float(a / hi), float(b / hi ** 3), float(c / hi ** 5)), float(E)


def quintic_image(coef, lo: float, hi: float) -> Tuple[float, float]:
    """Minimum and maximum of the odd quintic over [lo, hi]."""
    xs = np.linspace(lo, hi, 20001)
    a, b, c = coef
    cands = [lo, hi]
    # p'(x) = a + 3 b x^2 + 5 c x^4: roots in x^2
    for y in np.roots([5.0 * c, 3.0 * b, a]) if c != 0 else np.roots([3.0 * b, a]):
        if abs(y.imag) < 1e-12 and y.real > 0:
            r = float(np.sqrt(y.real))
            if lo < r < hi:
                cands.append(r)
    vals = np.concatenate([_p(coef, xs), _p(coef, np.array(cands))])
    return float(vals.min()), float(vals.max())


def polar_express_lp(lower: float, steps: int, safety: float = 1.0) -> Tuple[List[Tuple[float, float, float]], List[float]]:
    """Per-step (a, b, c) of the greedy minimax schedule and each step's max |1 - p| on its interval."""
    lo, hi = float(lower), 1.0
    coeffs, errs = [], []
    s = float(safety)
    for _ in range(steps):
        if hi - lo < 1e-3:
            a, b, c = FIXED_POINT_QUINTIC
        else:
            (a, b, c), _ = minimax_quintic_lp(lo, hi)
        q = (a / s, b / s ** 3, c / s ** 5)
        mn, mx = quintic_image(q, lo, hi)
        coeffs.append(q)
        errs.append(max(abs(1.0 - mn), abs(mx - 1.0)))
        lo, hi = mn, mx
    return coeffs, errs
