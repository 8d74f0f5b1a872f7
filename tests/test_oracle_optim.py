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


# ---------------------------------------------------------------- NorMuon

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("shape", [(16, 48), (48, 16), (24, 24)])
def test_normuon_keeps_frobenius_norm(shape):
    O = _rand(shape, 1)
    V = np.abs(_rand((min(shape),) if shape[0] != shape[1] else (shape[0],), 2))
    Op, _ = oo.normuon(O, V, 0.95)
    assert abs(np.linalg.norm(Op) / np.linalg.norm(O) - 1) < 1e-12


@pytest.mark.parametrize("shape", [(16, 48), (48, 16), (24, 24)])
def test_normuon_without_memory_equalises_neurons(shape):
    # beta2 = 0: V is this step's mean square, so every neuron of O' ends with
    # the same mean square over the reduction axis
    O = _rand(shape, 3) * np.linspace(0.1, 3.0, shape[1])[None, :] * np.linspace(0.5, 2.0, shape[0])[:, None]
    Op, V = oo.normuon(O, np.zeros(min(shape) if shape[0] != shape[1] else shape[0]), 0.0)
    ax = oo.normuon_axis(*shape)
    ms = np.mean(Op * Op, axis=ax)
    assert np.allclose(ms, ms.mean(), rtol=1e-12)
    assert np.allclose(V, np.mean(O * O, axis=ax), rtol=1e-14)


def test_normuon_is_identity_on_a_semi_orthogonal_update():
    # rows of a semi-orthogonal O (r <= c) have equal norms: nothing to equalise
    Q, _ = np.linalg.qr(_rand((40, 12), 4))
    O = Q.T                               # 12 x 40, O O^T = I
    Op, _ = oo.normuon(O, np.zeros(12), 0.95)
    assert np.allclose(Op, O, atol=1e-12)


def test_normuon_axis_follows_the_longer_side():
    O = _rand((12, 40), 5)
    V = np.abs(_rand((12,), 6))
    a, Va = oo.normuon(O, V, 0.9)
    b, Vb = oo.normuon(O.T, V, 0.9)
    assert np.allclose(a, b.T, atol=1e-14) and np.allclose(Va, Vb, atol=1e-14)


def test_normuon_second_moment_is_an_ema():
    O1, O2 = _rand((8, 20), 7), _rand((8, 20), 8)
    _, V1 = oo.normuon(O1, np.zeros(8), 0.9)
    _, V2 = oo.normuon(O2, V1, 0.9)
    m1, m2 = np.mean(O1 * O1, axis=1), np.mean(O2 * O2, axis=1)
    assert np.allclose(V2, 0.9 * 0.1 * m1 + 0.1 * m2, rtol=1e-14)


def test_normuon_scales_by_the_clamped_inverse_root():
    # two neurons with V = 4 and V = 1: the second is doubled relative to the first
    O = np.ones((2, 6))
    Op, _ = oo.normuon(O, np.array([4.0, 1.0]), 1.0)   # beta2 = 1 keeps V
    assert abs(Op[1, 0] / Op[0, 0] - 2.0) < 1e-12
    # a vanishing second moment is clamped at 1e-10, not divided by zero
    Oz, _ = oo.normuon(np.zeros((2, 6)), np.zeros(2), 0.5)
    assert np.all(np.isfinite(Oz)) and np.all(Oz == 0)


def test_muon_step_with_normuon_applies_it_after_newton_schulz():
    G = _rand((16, 48), 9)
    W = _rand((16, 48), 10) * 0.02
    W1, mom, V = oo.muon_step(W, G, np.zeros_like(G), lr=0.02, normuon_V=np.zeros(16), normuon_beta2=0.95)
    O = oo.newton_schulz(G)
    Op, Vref = oo.normuon(O, np.zeros(16), 0.95)
    assert np.allclose(W1, W - 0.02 * oo.muon_scale(16, 48) * Op, atol=1e-14)
    assert np.allclose(V, Vref, atol=1e-16)
