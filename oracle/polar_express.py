"""Offline generator for a Polar-Express-style Newton-Schulz coefficient table.

TEST INFRASTRUCTURE ONLY (see oracle/muon_oracle.py): it writes an input
table; the CUDA library never imports it.

PR #1396 "Record: Combined 3-Layer Recurrence + Parallel Residuals + Polar
Express + Brotli", table "Techniques Combined", row "Polar Express
Newton-Schulz", names a 4-step schedule of minimax-optimal quintic steps but
prints no coefficients.  This module builds such a table from the method's
published idea (Amsel, Persson, Musco & Gower, 2025: "The Polar Express"):
greedily, step by step, choose the odd quintic p(x) = a x + b x^3 + c x^5
that minimises max |1 - p(x)| over the interval [lo, hi] currently known to
hold the singular values, then move to the interval p maps it onto.

The minimax problem is solved by the Remez exchange algorithm in fp64:
{x, x^3, x^5} is a Chebyshev system on (0, inf), so the best approximation
equioscillates on 4 points including both end points.  The tests check the
equioscillation (the optimality certificate) directly.

Nothing here is copied from a printed table; the numbers come out of this
routine.  The table is an input to the optimizer: parity never depends on its
values.
"""

from __future__ import annotations

import numpy as np

__all__ = ["minimax_odd_quintic", "polar_express_table", "composed_band"]


def _solve_reference(xs: np.ndarray) -> tuple[np.ndarray, float]:
    """Solve p(x_i) + (-1)^i E = 1 on 4 reference points for (a, b, c, E)."""
    A = np.zeros((4, 4))
    for i, x in enumerate(xs):
        A[i, 0] = x
        A[i, 1] = x ** 3
        A[i, 2] = x ** 5
        A[i, 3] = (-1.0) ** i
    sol = np.linalg.solve(A, np.ones(4))
    return sol[:3], float(sol[3])


def _interior_extrema(coef: np.ndarray, lo: float, hi: float) -> np.ndarray:
    """Critical points of p on (lo, hi): roots of a + 3b y + 5c y^2 = 0 with
    y = x^2."""
    a, b, c = coef
    ys = np.roots([5.0 * c, 3.0 * b, a]) if c != 0 else np.array([-a / (3.0 * b)])
    xs = []
    for y in np.atleast_1d(ys):
        if abs(np.imag(y)) > 1e-14 or np.real(y) <= 0:
            continue
        x = float(np.sqrt(np.real(y)))
        if lo < x < hi:
            xs.append(x)
    return np.array(sorted(xs))


def minimax_odd_quintic(lo: float, hi: float, iters: int = 100,
                        tol: float = 1e-15):
    """Best uniform approximation of the constant 1 on [lo, hi] by an odd
    quintic.  Returns ((a, b, c), E, reference points) where E is the minimax
    error; p maps [lo, hi] into [1 - E, 1 + E]."""
    if not (0.0 < lo < hi):
        raise ValueError("need 0 < lo < hi")
    # Chebyshev-like start on [lo, hi].
    t = np.cos(np.pi * np.arange(3, -1, -1) / 3.0)
    xs = lo + (hi - lo) * (t + 1.0) / 2.0
    coef, E = _solve_reference(xs)
    for _ in range(iters):
        ext = _interior_extrema(coef, lo, hi)
        if len(ext) != 2:
            break
        new = np.array([lo, ext[0], ext[1], hi])
        coef_new, E_new = _solve_reference(new)
        done = np.max(np.abs(new - xs)) <= tol * hi
        xs, coef, E = new, coef_new, E_new
        if done:
            break
    return (float(coef[0]), float(coef[1]), float(coef[2])), float(E), xs


def _image(coef, lo: float, hi: float) -> tuple[float, float]:
    """Exact range of p over [lo, hi]: end points and interior critical
    points."""
    a, b, c = coef
    xs = [lo, hi] + list(_interior_extrema(np.array(coef), lo, hi))
    ys = [a * x + b * x ** 3 + c * x ** 5 for x in xs]
    return min(ys), max(ys)


def polar_express_table(steps: int = 4, lo: float = 1e-3, hi: float = 1.0,
                        cushion: float = 0.0, inflate: float = 1.0):
    """Greedy per-step minimax schedule.

    Step k is the minimax odd quintic on the design interval
    [max(lo_k, cushion * hi_k), inflate * hi_k]; the next interval
    [lo_{k+1}, hi_{k+1}] is the exact image of [lo_k, hi_k] under it.
    cushion > 0 keeps the design away from tiny lower ends (whose optimal
    polynomials are steep, so bf16 rounding is amplified); inflate > 1 keeps
    values slightly above the nominal upper end inside the region the
    polynomial was designed for.  Both are stability margins of the same
    kind the method uses; cushion = 0, inflate = 1 is the plain greedy
    schedule.

    Returns (rows of (a, b, c), nominal intervals, design intervals)."""
    rows, intervals, design = [], [], []
    for _ in range(steps):
        intervals.append((lo, hi))
        d_lo, d_hi = max(lo, cushion * hi), inflate * hi
        design.append((d_lo, d_hi))
        coef, _, _ = minimax_odd_quintic(d_lo, d_hi)
        rows.append(coef)
        lo, hi = _image(coef, lo, hi)
    return rows, intervals, design


def composed_band(rows, lo: float, hi: float) -> tuple[float, float]:
    """Exact range of the composed schedule p_K o ... o p_1 over [lo, hi]:
    each step's exact image (end points and interior critical points) is the
    next step's domain."""
    for coef in rows:
        lo, hi = _image(coef, lo, hi)
    return lo, hi
