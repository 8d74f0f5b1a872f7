"""The Newton-Schulz entry point that allocates no device memory.

Callers whose device memory is owned by another allocator, or who cannot
pass device scratch, use gpt_op_newton_schulz_noalloc: its scratch is a
fixed array inside the loaded library.  This file is collected last so a
stop-at-first-failure run has exercised everything else first; it also runs
alone in a fresh process.
"""
import numpy as np
import pytest

import synthetic as syn

pytestmark = pytest.mark.gpu

MUON_RELFRO = 2e-2   # the Muon update tolerance the other tests use


def _relfro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_noalloc_matches_allocating_entry_point_on_consecutive_calls():
    import torch

    import gpt_pretraining_step_b200 as g
    g.lib()
    # two different inputs, one call each, back to back on the shared array
    shapes = [(3, 256, 320), (2, 384, 128)]
    for i, shape in enumerate(shapes):
        G = torch.tensor(syn.gaussian(shape, seed=500 + i)).cuda()
        ref = g.newton_schulz(G, tf32_steps=3)
        got = g.newton_schulz_noalloc(G, tf32_steps=3)
        torch.cuda.synchronize()
        err = _relfro(got.double().cpu().numpy(), ref.double().cpu().numpy())
        assert err <= MUON_RELFRO, (shape, err)


def test_noalloc_rejects_inputs_beyond_its_limit():
    import torch

    import gpt_pretraining_step_b200 as g
    G = torch.zeros((1, 1024, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(g.GptError) as e:
        g.newton_schulz_noalloc(G)
    assert e.value.code == g.GPT_EINVAL
    assert "262144" in str(e.value)
