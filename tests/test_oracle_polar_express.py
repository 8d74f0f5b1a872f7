"""Pins of the Polar Express coefficient construction (CPU only)."""
import os

import numpy as np
import pytest

from oracle import polar_express as pe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "polar_express_printed.txt")


def _printed():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    return np.array([[float(v) for v in r] for r in rows])


def test_reproduces_printed_tuples():
    # the pages print three decimals; the construction must agree to +-0.001
    table = np.array(pe.coefficients())
    printed = _printed()
    assert printed.shape == (2, 3)
    assert np.max(np.abs(table[:2] - printed)) <= 1e-3


def test_five_steps():
    assert len(pe.coefficients()) == 5


@pytest.mark.parametrize("lo,hi", [(1e-3, 1.0), (0.02, 1.0), (0.3, 1.7), (0.9, 1.1)])
def test_minimax_equioscillates(lo, hi):
    a, b, c, e = pe.minimax_odd_quintic(lo, hi)
    x = np.linspace(lo, hi, 200001)
    err = pe.quintic((a, b, c), x) - 1.0
    # Chebyshev alternation: the max error is attained with alternating sign
    assert abs(np.max(np.abs(err)) - abs(e)) <= 1e-9 * max(1.0, abs(e))
    assert pe.quintic((a, b, c), lo) == pytest.approx(1.0 - e, abs=1e-12)
    assert pe.quintic((a, b, c), hi) == pytest.approx(1.0 + e, abs=1e-12)
    # any perturbation of the coefficients is worse in max norm
    rng = np.random.default_rng(0)
    for _ in range(20):
        d = rng.standard_normal(3) * 1e-4
        err2 = pe.quintic((a + d[0], b + d[1], c + d[2]), x) - 1.0
        assert np.max(np.abs(err2)) >= np.max(np.abs(err)) - 1e-12


def test_near_one_limit_is_textbook_quintic():
    # as the interval shrinks onto 1 the optimal quintic tends to the classical
    # Newton-Schulz quintic (15/8, -10/8, 3/8): p(1) = 1, p'(1) = p''(1) = 0
    a, b, c, _ = pe.minimax_odd_quintic(1 - 1e-3, 1 + 1e-3)
    assert np.allclose([a, b, c], [15 / 8, -10 / 8, 3 / 8], atol=1e-4)


def test_composition_maps_interval_into_band():
    table = pe.coefficients()
    x = np.geomspace(1e-3, 1.0, 10001)
    y = pe.composed(table, x)
    # every singular value in [1e-3, 1] lands in a narrow band around 1
    assert y.min() > 0.6 and y.max() < 1.25
    # the band is exactly the image interval the construction tracks
    lo = 1e-3
    for coef in table:
        lo = pe.quintic(coef, lo)
    assert y.min() == pytest.approx(lo, rel=1e-6)
