"""Pins of the fp64 Muon / AdamW oracle (CPU only)."""
import numpy as np
import pytest

from oracle import optim as oo
from oracle import polar_express as pe


def _svd_closed_form(G, table):
    # Newton-Schulz with odd polynomials acts on singular values only:
    # NS(G) = U f(S / ||G||_F) V^T with f the composed scalar map
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    fs = pe.composed(table, S / (np.linalg.norm(G) + oo.NS_EPS))
    return (U * fs) @ Vt


@pytest.mark.parametrize("shape", [(16, 40), (40, 16), (32, 32), (7, 129)])
def test_newton_schulz_matches_svd(shape):
    rng = np.random.default_rng(sum(shape))
    G = rng.standard_normal(shape)
    table = pe.coefficients()
    X = oo.newton_schulz(G, table)
    ref = _svd_closed_form(G, table)
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 1e-10


def test_newton_schulz_ill_conditioned():
    rng = np.random.default_rng(7)
    U, _ = np.linalg.qr(rng.standard_normal((24, 24)))
    V, _ = np.linalg.qr(rng.standard_normal((60, 60)))
    S = np.geomspace(1.0, 1e-6, 24)
    G = (U * S) @ V[:24]
    table = pe.coefficients()
    X = oo.newton_schulz(G, table)
    assert np.linalg.norm(X - _svd_closed_form(G, table)) / np.linalg.norm(X) < 1e-10


def test_newton_schulz_singular_values_in_band():
    # for singular values in [1e-3, 1] of the normalised input the output ones
    # land in the band of the composed map (near 1)
    rng = np.random.default_rng(11)
    G = rng.standard_normal((64, 256))
    table = pe.coefficients()
    s = np.linalg.svd(oo.newton_schulz(G, table), compute_uv=False)
    band = pe.composed(table, np.geomspace(1e-3, 1.0, 20001))
    assert s.min() >= band.min() - 1e-12 and s.max() <= band.max() + 1e-12


def test_newton_schulz_is_scale_free():
    rng = np.random.default_rng(12)
    G = rng.standard_normal((20, 50))
    # exact up to the 1e-7 added to the norm, amplified by the steep first steps
    X1, X2 = oo.newton_schulz(G), oo.newton_schulz(1e3 * G)
    assert np.linalg.norm(X1 - X2) / np.linalg.norm(X1) < 1e-6


def test_muon_first_step_convention_free():
    # Mom starts at zero, so Mom_1 = G for any beta; Frobenius normalisation
    # removes the (1 - beta) factor an EMA convention would add
    rng = np.random.default_rng(13)
    W = rng.standard_normal((24, 72)) * 0.02
    G = rng.standard_normal((24, 72))
    W1, _ = oo.muon_step(W, G, np.zeros_like(G), lr=0.02, momentum=0.95)
    W2, _ = oo.muon_step(W, 0.05 * G, np.zeros_like(G), lr=0.02, momentum=0.5)
    assert np.linalg.norm(W1 - W2) / np.linalg.norm(W1 - W) < 1e-6


def test_muon_update_scale_and_weight_decay():
    rng = np.random.default_rng(14)
    for rows, cols, s in [(24, 72, 1.0), (96, 24, 2.0)]:
        W = rng.standard_normal((rows, cols)) * 0.02
        G = rng.standard_normal((rows, cols))
        lr, wd = 0.02, 0.1
        W1, mom = oo.muon_step(W, G, np.zeros_like(G), lr=lr, weight_decay=wd)
        O = oo.newton_schulz(G)
        assert np.allclose(W1, W * (1 - lr * wd) - lr * s * O, atol=1e-15)
        assert np.array_equal(mom, G)


def test_adamw_first_step_closed_form():
    # bias correction makes m_hat = g and v_hat = g^2 at step 1, for any betas
    rng = np.random.default_rng(15)
    p = rng.standard_normal(1000)
    g = rng.standard_normal(1000) * 1e-3
    for b1, b2 in [(0.8, 0.95), (0.9, 0.999)]:
        p1, m, v = oo.adamw_step(p, g, np.zeros_like(g), np.zeros_like(g), 1,
                                 lr=3e-3, beta1=b1, beta2=b2, eps=1e-10, weight_decay=0.1)
        assert np.allclose(p1, p * (1 - 3e-3 * 0.1) - 3e-3 * g / (np.abs(g) + 1e-10),
                           atol=1e-15)


def test_adamw_constant_gradient_every_step():
    # a constant gradient keeps m_hat = g and v_hat = g^2 at every step
    rng = np.random.default_rng(16)
    g = rng.standard_normal(100)
    p = np.zeros(100); m = np.zeros(100); v = np.zeros(100)
    for t in range(1, 6):
        p_prev = p
        p, m, v = oo.adamw_step(p, g, m, v, t, lr=1e-2, eps=0.0)
        assert np.allclose(p - p_prev, -1e-2 * np.sign(g), atol=1e-13)
