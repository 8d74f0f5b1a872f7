"""fp64 Muon and AdamW updates (plain numpy).

TEST INFRASTRUCTURE ONLY: see the package header.

Routing ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador
Muon", parameter table): embeddings and lm_head go to AdamW, the 2-D block
matrices to Muon.

Muon ("Como Treinar Seu Próprio ChatGPT por 50 Dólares?", section "2. O
Otimizador Muon": momentum orthogonalised by a quintic Newton-Schulz
iteration, the Polar Express loop X <- aX + X(bA + cA^2), A = X^T X).  The
loop is written here on the smaller Gram side, A = X X^T and X <- aX + (bA +
cA^2) X with X transposed so that rows <= cols, which is the same map.
Readings where the pages are silent: momentum Mom <- beta Mom + G (no
Nesterov), input normalised by its Frobenius norm plus 1e-7, update
W <- W (1 - lr wd) - lr sqrt(max(1, rows/cols)) NS(Mom).

NorMuon ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "2. Optimizador
Muon", the "Reducción de varianza NorMuon" snippet, which is garbled: its
reduction axis and v_norm_new are undefined).  Reading: the orthogonalised
update O gets a per-neuron second moment, the mean of O^2 over the longer
axis (the columns for a square matrix), kept as an EMA V <- b2 V + (1 - b2)
v_mean with V = 0 before the first step; O is multiplied by V^(-1/2)
(V clamped at 1e-10) along the shorter axis and rescaled so that the result
keeps O's Frobenius norm (v_norm / v_norm_new with the same mean-of-squares
norm before and after, the denominator clamped at 1e-10).

AdamW: the textbook decoupled-weight-decay update with bias correction.
"""
from __future__ import annotations

import numpy as np

from .polar_express import coefficients

NS_EPS = 1e-7


def newton_schulz(G, table=None):
    """Polar Express iteration on G / (||G||_F + eps); any shape, fp64."""
    table = coefficients() if table is None else table
    X = np.asarray(G, dtype=np.float64)
    X = X / (np.linalg.norm(X) + NS_EPS)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    for a, b, c in table:
        A = X @ X.T
        Bm = b * A + c * (A @ A)
        X = a * X + Bm @ X
    return X.T if transposed else X


def muon_scale(rows, cols):
    return float(np.sqrt(max(1.0, rows / cols)))


def normuon_axis(rows, cols):
    """Axis the NorMuon second moment averages over: the longer one (columns
    for a square matrix)."""
    return 0 if rows > cols else 1


def normuon(O, V, beta2=0.95):
    """Returns (O', V') for the orthogonalised update O [rows, cols] and the
    per-neuron second-moment EMA V (one entry per row, or per column when
    rows > cols)."""
    O = np.asarray(O, dtype=np.float64)
    ax = normuon_axis(*O.shape)
    v_mean = np.mean(O * O, axis=ax)
    V = beta2 * np.asarray(V, dtype=np.float64) + (1.0 - beta2) * v_mean
    s = 1.0 / np.sqrt(np.maximum(V, 1e-10))
    v_norm = np.sqrt(np.sum(v_mean))
    v_norm_new = np.sqrt(np.sum(v_mean * s * s))
    f = s * (v_norm / max(v_norm_new, 1e-10))
    Oprime = O * (f[None, :] if ax == 0 else f[:, None])
    return Oprime, V


def muon_step(W, G, mom, lr, momentum=0.95, weight_decay=0.0, table=None, normuon_V=None, normuon_beta2=0.95):
    """Returns (W', mom') for one [rows, cols] matrix, or (W', mom', V') with
    the NorMuon variance reduction when its state normuon_V is given."""
    W = np.asarray(W, dtype=np.float64)
    mom = momentum * np.asarray(mom, dtype=np.float64) + np.asarray(G, dtype=np.float64)
    O = newton_schulz(mom, table)
    if normuon_V is not None:
        O, V = normuon(O, normuon_V, normuon_beta2)
    rows, cols = W.shape
    W = W * (1.0 - lr * weight_decay) - lr * muon_scale(rows, cols) * O
    return (W, mom) if normuon_V is None else (W, mom, V)


def adamw_step(p, g, m, v, step, lr, beta1=0.8, beta2=0.95, eps=1e-10,
               weight_decay=0.0):
    """Returns (p', m', v') after step number ``step`` (1-based)."""
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    p = p * (1.0 - lr * weight_decay) - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v
