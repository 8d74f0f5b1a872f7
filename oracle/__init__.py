"""fp64 CPU oracle of one GPT pretraining step.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline may import this package.  The CUDA library never calls it and shares
no code with it; the one module both sides use is ``synthetic`` (seeded input
generation, none of the method's arithmetic).

Sources: the pages "¿Cómo Entrenar Tu Propio ChatGPT por $50?" and "Como
Treinar Seu Próprio ChatGPT por 50 Dólares?" (sections "1. Modelo GPT",
"2. Optimizador Muon", "3. Gestión de Precisión").  Each module cites the
passage it follows and lists the readings it takes where the pages are
silent.

Pins (tests/test_oracle_*.py, all CPU):
  model.py          finite-difference gradients of every tensor; loss = ln V
                    exactly when lm_head is zero; initial loss against the
                    Gaussian closed form ln V + sigma^2/2; causality; RoPE
                    norm and relative-position invariants; attention special
                    cases (one position, equal keys).
  polar_express.py  the two tuples the pages print; equioscillation of each
                    minimax quintic.
  optim.py          Newton-Schulz against the SVD closed form U f(S) V^T;
                    AdamW step-1 closed form; Muon step-1 independence of the
                    momentum convention; weight-decay scaling.
  fp8.py            the e4m3 grid (every representable value, saturation and
                    ties-to-even), checked against the format definition.
"""
from . import fp8, model, optim, polar_express  # noqa: F401
