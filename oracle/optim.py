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


def muon_step(W, G, mom, lr, momentum=0.95, weight_decay=0.0, table=None):
    """Returns (W', mom') for one [rows, cols] matrix."""
    W = np.asarray(W, dtype=np.float64)
    mom = momentum * np.asarray(mom, dtype=np.float64) + np.asarray(G, dtype=np.float64)
    O = newton_schulz(mom, table)
    rows, cols = W.shape
    W = W * (1.0 - lr * weight_decay) - lr * muon_scale(rows, cols) * O
    return W, mom


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
