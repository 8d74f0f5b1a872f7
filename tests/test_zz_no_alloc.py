"""The Newton-Schulz entry point that allocates no device memory.

Some callers cannot give this library device scratch: their device memory
belongs to another allocator (a framework's caching pool that has already
reserved the GPU), their runtime forbids cudaMalloc after start-up, or their
interface has no place for a scratch pointer.  gpt_op_newton_schulz_noalloc
keeps its scratch in a fixed array inside the loaded library instead.  These
tests compare it with the fp64 oracle's Newton-Schulz (and with the
allocating entry point) on two calls in a row that share the array, and
check its size limit.  This file is collected last, so a run that stops at
the first failure has exercised everything else first; it also passes run
alone in a fresh process.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import optim as oo

pytestmark = pytest.mark.gpu

MUON_RELFRO = 2e-2   # the Muon update tolerance the other tests use


def _relfro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("tf32_steps", [-1, 3])
def test_noalloc_matches_oracle_on_consecutive_calls(tf32_steps):
    import torch

    import gpt_pretraining_step_b200 as g
    g.lib()
    # two different inputs, one call each, back to back on the shared array;
    # the second is wider than tall (the transposed path)
    shapes = [(3, 256, 320), (2, 384, 128)]
    for i, shape in enumerate(shapes):
        G = syn.gaussian(shape, seed=500 + i)
        tG = torch.tensor(G).cuda()
        got = g.newton_schulz_noalloc(tG, tf32_steps=tf32_steps)
        ref_gpu = g.newton_schulz(tG, tf32_steps=tf32_steps)
        g.op_check()
        got64 = got.double().cpu().numpy()
        for z in range(shape[0]):
            ref = oo.newton_schulz(G[z].astype(np.float64))
            err = _relfro(got64[z], ref)
            assert err <= MUON_RELFRO, (shape, z, err)
        assert _relfro(got64, ref_gpu.double().cpu().numpy()) <= MUON_RELFRO, shape


def test_noalloc_rejects_inputs_beyond_its_limit():
    import torch

    import gpt_pretraining_step_b200 as g
    G = torch.zeros((1, 1024, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(g.GptError) as e:
        g.newton_schulz_noalloc(G)
    assert e.value.code == g.GPT_EINVAL
    assert "262144" in str(e.value)
