"""All the options of the step in one model (B200 only): grouped kv heads,
a per-layer window pattern, the residual extras and value embeddings through
forward and backward, then a NorMuon and an AdamW step, against the fp64
oracle at the whole-step tolerances (loss relative error <= 1e-2, gradient
cosine >= 0.999, Muon update relative Frobenius error <= 2e-2)."""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as om
from oracle import optim as oo

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-2
GRAD_COS = 0.999
MUON_RELFRO = 2e-2


@pytest.fixture(scope="module")
def torch():
    import torch as t
    import gpt_pretraining_step_b200 as g
    g.lib()
    return t


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def cosine(a, b):
    a, b = np.ravel(a), np.ravel(b)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def relfro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def test_every_option_together_matches_oracle(torch):
    """Grouped kv heads, an "SSL" window pattern, the residual extras and
    value embeddings in one model, then a NorMuon step and an AdamW step."""
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=3, d_model=512, vocab=704, batch=2, seq_len=384, n_kv_head=2)
    params = syn.init_params(s, seed=71, extras=True, ve_channels=8)
    params["ve_gate"] = syn.gaussian(params["ve_gate"].shape, seed=72, std=2.0)
    params["scalars"] = syn.random_scalars(s, seed=73)
    tok, tgt = syn.tokens(s, seed=74), syn.targets(s, seed=75)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   residual_extras=True, ve_gate_channels=8, n_kv_head=2, window_pattern="SSL", short_window=150)
    specs = syn.param_specs(s, extras=True, ve_channels=8)
    for tid, (pname, *_r) in enumerate(specs):
        st.set(tid, params[pname])
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    windows = om.layer_windows("SSL", 150, s.depth)
    loss_ref, grads, _ = om.fwd_bwd(params, tok, tgt, s.depth, windows=windows)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    G = {}
    for tid, (pname, *_r) in enumerate(specs):
        G[pname] = f64(st.get(tid, g.KIND_GRAD))
        cs = cosine(G[pname], grads[pname])
        assert cs >= GRAD_COS, (pname, cs)
    st.muon_step_normuon(0.02, 0.95, 0.01, 0.9)
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        W0 = params[pname].astype(np.float64)
        if grp == "muon":
            W_ref, _, _ = oo.muon_step(W0, G[pname], np.zeros((r, c)), 0.02, 0.95, 0.01,
                                       normuon_V=np.zeros(min(r, c)), normuon_beta2=0.9)
            assert relfro(f64(st.get(tid, g.KIND_PARAM)) - W0, W_ref - W0) <= MUON_RELFRO, pname
        else:
            W_ref, _, _ = oo.adamw_step(W0, G[pname], np.zeros((r, c)), np.zeros((r, c)), 1, 3e-3, 0.8, 0.95,
                                        1e-10, 0.0)
            assert np.abs(f64(st.get(tid, g.KIND_PARAM)) - W_ref).max() < 1e-6, pname


def test_checkpoint_restores_the_step_exactly(torch):
    """state_dict / load_state_dict (every value, momentum, NorMuon and AdamW
    state and the AdamW step count) give a fresh context the same next step."""
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=2, d_model=256, vocab=1000, batch=2, seq_len=200)
    params = syn.init_params(s, seed=81, extras=True, ve_channels=8)
    cfg = dict(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
               residual_extras=True, ve_gate_channels=8)
    specs = syn.param_specs(s, extras=True, ve_channels=8)
    # the first context runs on a stream of its own: a checkpoint read from it
    # must still see every copy completed (the binding orders them before
    # torch's current stream)
    side = torch.cuda.Stream()
    a = g.GPTStep(**cfg, stream=side)
    for tid, (pname, *_r) in enumerate(specs):
        a.set(tid, params[pname])
    batches = [(torch.tensor(syn.tokens(s, seed=82 + 2 * i)).cuda(), torch.tensor(syn.targets(s, seed=83 + 2 * i)).cuda())
               for i in range(2)]

    def step(st, tok, tgt):
        loss = float(st.fwd_bwd(tok, tgt).item())
        st.muon_step_normuon(0.02, 0.95, 0.01, 0.9)
        st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.01)
        st.check()
        return loss

    step(a, *batches[0])
    state = a.state_dict()
    assert state["adam_step"] == 1
    b = g.GPTStep(**cfg)
    b.load_state_dict(state)
    again = b.state_dict()
    assert again["adam_step"] == 1 and again["tensors"].keys() == state["tensors"].keys()
    for key, value in state["tensors"].items():
        assert np.array_equal(again["tensors"][key], value), key
    la, lb = step(a, *batches[1]), step(b, *batches[1])
    assert la == lb                                   # identical weights: the same forward, bit for bit
    for tid, (pname, *_r) in enumerate(specs):
        # the attention backward adds dq partial sums in no fixed order, so the
        # updates agree to rounding
        assert np.allclose(f64(a.get(tid)), f64(b.get(tid)), rtol=1e-5, atol=1e-7), pname
