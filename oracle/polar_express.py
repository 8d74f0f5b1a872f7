"""Polar Express coefficients for the Muon Newton-Schulz iteration (fp64).

TEST INFRASTRUCTURE ONLY: see the package header.

"¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador Muon"
(the Polar Express snippet) prints the first two (a, b, c) tuples of a
five-step table to three decimals and elides the rest.  The table is the
output of the Polar Express construction (Amsel, Persson, Musco and Gower,
2025): at every step pick the odd quintic p(x) = a x + b x^3 + c x^5 that is
the minimax approximation of the constant 1 on the current interval [l, u]
(its error equioscillates at four points), clamp the lower end to a cushion
fraction of u so that the steep first polynomial stays tame, recentre it so
that 1 - p(l) = p(u) - 1 on the true interval, shrink it by a safety factor
s (p(x) -> p(x / s), which keeps bf16 rounding from pushing singular values
past the basin of the next step) and carry the image interval
[p(l), 2 - p(l)] to the next step.

Reading of the pages: l0 = 1e-3, cushion = 0.02 and safety factor 1.02
reproduce both printed tuples to within their printed precision; the same
construction then fixes steps 3 to 5.  The pins are in
tests/test_oracle_polar_express.py (printed tuples, equioscillation).
"""
from __future__ import annotations

import numpy as np

L0 = 1e-3
CUSHION = 0.02
SAFETY = 1.02
STEPS = 5


def minimax_odd_quintic(lo: float, hi: float, iters: int = 200):
    """Odd quintic closest to 1 in max-norm on [lo, hi] (Remez exchange).

    Returns (a, b, c, E): p(lo) = 1 - E, p(q) = 1 + E, p(r) = 1 - E,
    p(hi) = 1 + E at the two interior extrema q < r.
    """
    q = lo + 0.3 * (hi - lo)
    r = lo + 0.7 * (hi - lo)
    sol = None
    for _ in range(iters):
        xs = np.array([lo, q, r, hi])
        lhs = np.stack([xs, xs ** 3, xs ** 5, np.array([1.0, -1.0, 1.0, -1.0])], axis=1)
        sol = np.linalg.solve(lhs, np.ones(4))
        a, b, c, _ = sol
        # interior extrema of p: roots of p'(x) = a + 3 b x^2 + 5 c x^4
        disc = 9.0 * b * b - 20.0 * a * c
        if disc < 0 or c == 0:
            break
        x2 = (-3.0 * b + np.array([-1.0, 1.0]) * np.sqrt(disc)) / (10.0 * c)
        if np.any(x2 <= 0):
            break
        nq, nr = np.sort(np.sqrt(x2))
        if abs(nq - q) < 1e-16 and abs(nr - r) < 1e-16:
            break
        q, r = nq, nr
    a, b, c, e = sol
    return float(a), float(b), float(c), float(e)


def quintic(coef, x):
    a, b, c = coef
    return a * x + b * x ** 3 + c * x ** 5


def coefficients(steps: int = STEPS, l0: float = L0, cushion: float = CUSHION,
                 safety: float = SAFETY):
    """The (a, b, c) table, one tuple per Newton-Schulz step."""
    lo, hi = l0, 1.0
    table = []
    for _ in range(steps):
        a, b, c, _ = minimax_odd_quintic(max(lo, cushion * hi), hi)
        centre = 2.0 / (quintic((a, b, c), lo) + quintic((a, b, c), hi))
        a, b, c = a * centre, b * centre, c * centre
        coef = (a / safety, b / safety ** 3, c / safety ** 5)
        table.append(coef)
        lo = quintic(coef, lo)
        hi = 2.0 - lo
    return table


def composed(table, x):
    """f = p_n o ... o p_1 applied to scalars (the spectral map of the iteration)."""
    y = np.asarray(x, dtype=np.float64)
    for coef in table:
        y = quintic(coef, y)
    return y
