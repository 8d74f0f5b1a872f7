"""Whole-step parity of libgpt against the fp64 oracle (B200 only).

Tolerances (stated for the step): loss relative error <= 1e-2, per-tensor
gradient cosine >= 0.999, Muon update relative Frobenius error <= 2e-2,
token/target indexing exact.  Small configurations run the full oracle;
the d20 configuration (the benchmark's launch shape) is checked on sampled
outputs the oracle computes one by one (per-position losses of a prefix,
single matrices of the optimizer) and on properties that hold at any size.
"""
import math

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


def build(torch, shape, params=None, ns_tf32_steps=-1, lm_chunk_rows=0):
    import gpt_pretraining_step_b200 as g
    st = g.GPTStep(depth=shape.depth, batch=shape.batch, seq_len=shape.seq_len, vocab=shape.vocab,
                   d_model=shape.d_model, ns_tf32_steps=ns_tf32_steps, lm_chunk_rows=lm_chunk_rows)
    if params is not None:
        for tid, (name, *_rest) in enumerate(syn.param_specs(shape)):
            st.set(tid, params[name])
    return st


SMALL = {
    "tiny": syn.config_shape("tiny"),
    # several 128-row tiles with a ragged tail, two heads, a vocab that is not a tile multiple
    "ragged": syn.make_shape(depth=2, d_model=256, vocab=1000, batch=2, seq_len=200),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_fwd_bwd_matches_oracle(torch, name):
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=0)
    tok, tgt = syn.tokens(s), syn.targets(s)
    # a small lm_head chunk exercises the chunked loss path on several chunks
    st = build(torch, s, params, lm_chunk_rows=128 if name == "ragged" else 0)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    loss_ref, grads, cache = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    row = f64(st.row_loss()).ravel()
    assert np.abs(row - cache["row_loss"]).max() < 2e-2
    for tid, (pname, *_r) in enumerate(syn.param_specs(s)):
        got = f64(st.get(tid, g.KIND_GRAD))
        c = cosine(got, grads[pname])
        assert c >= GRAD_COS, (pname, c)


@pytest.mark.parametrize("pattern,short_window", [("SSSL", 150), ("SL", 0), ("S", 128)])
def test_sliding_window_layers_match_oracle(torch, pattern, short_window):
    """Per-layer attention windows ("SSSL"-style pattern repeated over the
    layers) through the whole forward and backward."""
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=4, d_model=256, vocab=1000, batch=2, seq_len=520)
    params = syn.init_params(s, seed=21)
    tok, tgt = syn.tokens(s, seed=22), syn.targets(s, seed=23)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   window_pattern=pattern, short_window=short_window)
    for tid, (name, *_rest) in enumerate(syn.param_specs(s)):
        st.set(tid, params[name])
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    windows = om.layer_windows(pattern, short_window, s.depth)
    loss_ref, grads, cache = om.fwd_bwd(params, tok, tgt, s.depth, windows=windows)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    assert np.abs(f64(st.row_loss()).ravel() - cache["row_loss"]).max() < 2e-2
    for tid, (pname, *_r) in enumerate(syn.param_specs(s)):
        c = cosine(f64(st.get(tid, g.KIND_GRAD)), grads[pname])
        assert c >= GRAD_COS, (pname, c)


def _build_extras(torch, s, params):
    import gpt_pretraining_step_b200 as g
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   residual_extras=True)
    for tid, (name, *_rest) in enumerate(syn.param_specs(s, extras=True)):
        st.set(tid, params[name])
    return st


def test_neutral_residual_extras_are_bit_identical_to_plain(torch):
    """Scales 1 / 0 / 0 (the initial values) change nothing, bit for bit."""
    import gpt_pretraining_step_b200 as g
    s = SMALL["ragged"]
    params = syn.init_params(s, seed=41, extras=True)
    tok, tgt = torch.tensor(syn.tokens(s, seed=42)).cuda(), torch.tensor(syn.targets(s, seed=43)).cuda()
    plain = build(torch, s, params)
    ext = _build_extras(torch, s, params)
    assert ext.num_tensors() == plain.num_tensors() + 1
    assert torch.equal(ext.get(ext.num_tensors() - 1), torch.tensor(params["scalars"]).cuda())
    la = float(plain.fwd_bwd(tok, tgt).item())
    lb = float(ext.fwd_bwd(tok, tgt).item())
    plain.check()
    ext.check()
    assert la == lb
    for tid in range(plain.num_tensors()):
        assert torch.equal(plain.get(tid, g.KIND_GRAD), ext.get(tid, g.KIND_GRAD)), tid


@pytest.mark.parametrize("name", list(SMALL))
def test_residual_extras_match_oracle(torch, name):
    """Random residual / x0 / backout scales through the forward, the backward
    (the scalars' gradients included) and the AdamW step of the scalars."""
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=44, extras=True)
    params["scalars"] = syn.random_scalars(s, seed=45)
    tok, tgt = syn.tokens(s, seed=46), syn.targets(s, seed=47)
    st = _build_extras(torch, s, params)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    loss_ref, grads, cache = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    assert np.abs(f64(st.row_loss()).ravel() - cache["row_loss"]).max() < 2e-2
    specs = syn.param_specs(s, extras=True)
    for tid, (pname, *_r) in enumerate(specs):
        got = f64(st.get(tid, g.KIND_GRAD))
        c = cosine(got, grads[pname])
        assert c >= GRAD_COS, (pname, c)
    sid = len(specs) - 1
    gs = f64(st.get(sid, g.KIND_GRAD))
    assert relfro(gs, grads["scalars"]) <= 3e-2
    # AdamW moves the scalars like the oracle does given the same gradient
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()
    p_ref, _, _ = oo.adamw_step(params["scalars"].astype(np.float64), gs, np.zeros_like(gs), np.zeros_like(gs), 1,
                                3e-3, 0.8, 0.95, 1e-10, 0.0)
    assert np.abs(f64(st.get(sid, g.KIND_PARAM)) - p_ref).max() < 1e-6


VE_C = 16


def _build_ve(torch, s, params, extras=False):
    import gpt_pretraining_step_b200 as g
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   residual_extras=extras, ve_gate_channels=VE_C)
    for tid, (name, *_rest) in enumerate(syn.param_specs(s, extras=extras, ve_channels=VE_C)):
        st.set(tid, params[name])
    return st


def test_zero_value_embeddings_are_bit_identical_to_plain(torch):
    import gpt_pretraining_step_b200 as g
    s = SMALL["ragged"]
    params = syn.init_params(s, seed=51, ve_channels=VE_C)
    for l in syn.ve_layers(s.depth):
        params[f"ve{l}"] = np.zeros_like(params[f"ve{l}"])
    params["ve_gate"] = syn.gaussian(params["ve_gate"].shape, seed=52)
    tok, tgt = torch.tensor(syn.tokens(s, seed=53)).cuda(), torch.tensor(syn.targets(s, seed=54)).cuda()
    plain = build(torch, s, params)
    ve = _build_ve(torch, s, params)
    assert ve.num_tensors() == plain.num_tensors() + len(syn.ve_layers(s.depth)) + 1
    la = float(plain.fwd_bwd(tok, tgt).item())
    lb = float(ve.fwd_bwd(tok, tgt).item())
    plain.check()
    ve.check()
    assert la == lb
    for tid in range(plain.num_tensors()):
        assert torch.equal(plain.get(tid, g.KIND_GRAD), ve.get(tid, g.KIND_GRAD)), tid


@pytest.mark.parametrize("name,extras", [("tiny", False), ("ragged", False), ("ragged", True)])
def test_value_embeddings_match_oracle(torch, name, extras):
    """Random tables and gates (with and without the residual extras): loss,
    every gradient (tables and gates included), and the gates' AdamW step."""
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=55, extras=extras, ve_channels=VE_C)
    params["ve_gate"] = syn.gaussian(params["ve_gate"].shape, seed=56, std=2.0)
    if extras:
        params["scalars"] = syn.random_scalars(s, seed=57)
    tok, tgt = syn.tokens(s, seed=58), syn.targets(s, seed=59)
    st = _build_ve(torch, s, params, extras)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    loss_ref, grads, cache = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    assert np.abs(f64(st.row_loss()).ravel() - cache["row_loss"]).max() < 2e-2
    specs = syn.param_specs(s, extras=extras, ve_channels=VE_C)
    for tid, (pname, *_r) in enumerate(specs):
        c = cosine(f64(st.get(tid, g.KIND_GRAD)), grads[pname])
        assert c >= GRAD_COS, (pname, c)
    gid = len(specs) - 1
    gg = f64(st.get(gid, g.KIND_GRAD))
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()
    p_ref, _, _ = oo.adamw_step(params["ve_gate"].astype(np.float64), gg, np.zeros_like(gg), np.zeros_like(gg), 1,
                                3e-3, 0.8, 0.95, 1e-10, 0.0)
    assert np.abs(f64(st.get(gid, g.KIND_PARAM)) - p_ref).max() < 1e-6


GQA_SHAPES = {
    "ragged_kv1": syn.make_shape(depth=2, d_model=256, vocab=1000, batch=2, seq_len=200, n_kv_head=1),
    "four_heads_kv2": syn.make_shape(depth=3, d_model=512, vocab=512, batch=1, seq_len=320, n_kv_head=2),
}


@pytest.mark.parametrize("name,extras,ve", [("ragged_kv1", False, 0), ("four_heads_kv2", False, 0),
                                            ("four_heads_kv2", True, 16)])
def test_grouped_kv_model_matches_oracle(torch, name, extras, ve):
    """Grouped kv heads through the narrower q|k|v projection, its epilogue,
    the attention kernels (kv heads at their query-head rows), the dq|dk|dv
    assembly and, with it, value embeddings and the residual extras; then one
    Muon step on the narrower matrices."""
    import gpt_pretraining_step_b200 as g
    s = GQA_SHAPES[name]
    params = syn.init_params(s, seed=61, extras=extras, ve_channels=ve)
    if ve:
        params["ve_gate"] = syn.gaussian(params["ve_gate"].shape, seed=62, std=2.0)
    if extras:
        params["scalars"] = syn.random_scalars(s, seed=63)
    tok, tgt = syn.tokens(s, seed=64), syn.targets(s, seed=65)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   residual_extras=extras, ve_gate_channels=ve, n_kv_head=s.n_kv_head)
    specs = syn.param_specs(s, extras=extras, ve_channels=ve)
    assert st.num_tensors() == len(specs)
    for tid, (pname, r, c, grp) in enumerate(specs):
        assert st.tensor_info(tid)[:2] == (r, c), pname
        st.set(tid, params[pname])
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    loss_ref, grads, cache = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    assert np.abs(f64(st.row_loss()).ravel() - cache["row_loss"]).max() < 2e-2
    G = {}
    for tid, (pname, r, c, grp) in enumerate(specs):
        G[pname] = f64(st.get(tid, g.KIND_GRAD))
        cs = cosine(G[pname], grads[pname])
        assert cs >= GRAD_COS, (pname, cs)
    st.muon_step(0.02, 0.95, 0.0)
    st.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp != "muon":
            continue
        W0 = params[pname].astype(np.float64)
        W_ref, _ = oo.muon_step(W0, G[pname], np.zeros((r, c)), 0.02, 0.95, 0.0)
        assert relfro(f64(st.get(tid, g.KIND_PARAM)) - W0, W_ref - W0) <= MUON_RELFRO, pname


def test_embedding_and_target_indexing_exact(torch):
    # with a zero lm_head the logits vanish: loss = ln V exactly, and dW_lm has
    # one shared column for every vocabulary id that is not a target, so the set
    # of deviating columns must equal the set of targets; the embedding gradient
    # is non-zero exactly on the rows of the tokens present
    import gpt_pretraining_step_b200 as g
    s = SMALL["ragged"]
    params = syn.init_params(s, seed=1)
    params["lm_head"] = np.zeros_like(params["lm_head"])
    tok, tgt = syn.tokens(s, seed=11), syn.targets(s, seed=12)
    tok[0, :50] = 0
    tok[1, -3:] = s.vocab - 1
    tgt[0, 0] = 0
    tgt[1, 5] = s.vocab - 1
    st = build(torch, s, params)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    assert abs(loss - math.log(s.vocab)) < 1e-5
    G = f64(st.get(1, g.KIND_GRAD))
    absent = np.setdiff1d(np.arange(s.vocab), np.unique(tgt))
    base = G[:, absent[0]]
    dev = np.abs(G - base[:, None]).max(axis=0) > 1e-3 * np.abs(base).max()
    assert set(np.nonzero(dev)[0].tolist()) == set(np.unique(tgt).tolist())
    # a zero lm_head stops every gradient below it exactly
    assert np.abs(f64(st.get(0, g.KIND_GRAD))).max() == 0.0
    # with the trained-shape weights the embedding gradient is non-zero exactly
    # on the rows of the tokens present (ids 0 and V-1 included)
    params = syn.init_params(s, seed=1)
    st.set(1, params["lm_head"])
    st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda())
    st.check()
    E = f64(st.get(0, g.KIND_GRAD))
    nz = np.nonzero(np.abs(E).sum(axis=1) > 0)[0]
    assert set(nz.tolist()) == set(np.unique(tok).tolist())


def test_out_of_range_ids_are_reported_and_context_survives(torch):
    import gpt_pretraining_step_b200 as g
    s = SMALL["tiny"]
    st = build(torch, s, syn.init_params(s))
    tok, tgt = syn.tokens(s), syn.targets(s)
    bad = tok.copy()
    bad[1, 7] = s.vocab
    st.fwd_bwd(torch.tensor(bad).cuda(), torch.tensor(tgt).cuda())
    with pytest.raises(g.GptError) as e:
        st.check()
    assert e.value.code == g.GPT_ERANGE
    badt = tgt.copy()
    badt[0, 0] = -1
    st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(badt).cuda())
    with pytest.raises(g.GptError):
        st.check()
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    assert math.isfinite(loss)


def test_accumulate_doubles_gradients(torch):
    import gpt_pretraining_step_b200 as g
    s = SMALL["tiny"]
    st = build(torch, s, syn.init_params(s))
    tok, tgt = torch.tensor(syn.tokens(s)).cuda(), torch.tensor(syn.targets(s)).cuda()
    st.fwd_bwd(tok, tgt)
    g1 = [f64(st.get(t, g.KIND_GRAD)) for t in range(st.num_tensors())]
    st.fwd_bwd(tok, tgt, accumulate=True)
    st.check()
    for t in range(st.num_tensors()):
        g2 = f64(st.get(t, g.KIND_GRAD))
        assert relfro(g2, 2 * g1[t]) < 1e-5, t


def test_loss_is_deterministic(torch):
    s = SMALL["ragged"]
    st = build(torch, s, syn.init_params(s))
    tok, tgt = torch.tensor(syn.tokens(s)).cuda(), torch.tensor(syn.targets(s)).cuda()
    a = float(st.fwd_bwd(tok, tgt).item())
    b = float(st.fwd_bwd(tok, tgt).item())
    assert a == b


@pytest.mark.parametrize("name", list(SMALL))
def test_muon_step_matches_oracle(torch, name):
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=2)
    st = build(torch, s, params)
    specs = syn.param_specs(s)
    G = {}
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp == "muon":
            G[pname] = syn.gaussian((r, c), seed=100 + tid)
            st.set(tid, G[pname], kind=g.KIND_GRAD)
    lr, mom, wd = 0.02, 0.95, 0.01
    st.muon_step(lr, mom, wd)
    st.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp != "muon":
            continue
        W0 = params[pname].astype(np.float64)
        W_ref, mom_ref = oo.muon_step(W0, G[pname], np.zeros((r, c)), lr, mom, wd)
        W_got = f64(st.get(tid, g.KIND_PARAM))
        assert relfro(W_got - W0, W_ref - W0) <= MUON_RELFRO, pname
        assert np.allclose(f64(st.get(tid, g.KIND_MOM)), mom_ref, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("ns_tf32_steps", [-1, 5])
@pytest.mark.parametrize("name", list(SMALL))
def test_normuon_two_steps_match_oracle(torch, name, ns_tf32_steps):
    """Two NorMuon steps (the second exercises the second-moment EMA) against
    the oracle chain: each step's update, the momentum and the state V."""
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=7)
    st = build(torch, s, params, ns_tf32_steps=ns_tf32_steps)
    specs = syn.param_specs(s)
    lr, mom, wd, beta2 = 0.02, 0.95, 0.01, 0.9
    W = {p: params[p].astype(np.float64) for p, *_r in specs}
    M = {p: np.zeros((r, c)) for p, r, c, _g in specs}
    V = {p: np.zeros(min(r, c)) for p, r, c, _g in specs}
    for step in range(2):
        W_before = {tid: f64(st.get(tid, g.KIND_PARAM)) for tid in range(len(specs))}
        G = {}
        for tid, (pname, r, c, grp) in enumerate(specs):
            if grp == "muon":
                G[pname] = syn.gaussian((r, c), seed=300 + 10 * step + tid)
                st.set(tid, G[pname], kind=g.KIND_GRAD)
        st.muon_step_normuon(lr, mom, wd, beta2)
        st.check()
        for tid, (pname, r, c, grp) in enumerate(specs):
            if grp != "muon":
                continue
            W_prev = W[pname]
            W[pname], M[pname], V[pname] = oo.muon_step(W_prev, G[pname], M[pname], lr, mom, wd,
                                                        normuon_V=V[pname], normuon_beta2=beta2)
            got = f64(st.get(tid, g.KIND_PARAM))
            err = relfro(got - W_before[tid], W[pname] - W_prev)
            assert err <= MUON_RELFRO, (step, pname, err)
            assert np.allclose(f64(st.get(tid, g.KIND_MOM)), M[pname], rtol=1e-6, atol=1e-7)
            v_got = f64(st.get(tid, g.KIND_NORMUON_V))
            assert v_got.shape == V[pname].shape
            assert relfro(v_got, V[pname]) <= 2 * MUON_RELFRO, (step, pname)


def test_normuon_state_roundtrip_and_preset(torch):
    """A preset nonzero V enters the EMA; plain Muon leaves V untouched."""
    import gpt_pretraining_step_b200 as g
    s = SMALL["ragged"]
    params = syn.init_params(s, seed=8)
    st = build(torch, s, params)
    specs = syn.param_specs(s)
    rng = np.random.default_rng(9)
    V0, G = {}, {}
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp != "muon":
            continue
        V0[pname] = rng.uniform(1e-5, 1e-3, size=min(r, c))
        st.set(tid, V0[pname], kind=g.KIND_NORMUON_V)
        assert np.array_equal(f64(st.get(tid, g.KIND_NORMUON_V)), V0[pname].astype(np.float32))
        G[pname] = syn.gaussian((r, c), seed=400 + tid)
        st.set(tid, G[pname], kind=g.KIND_GRAD)
    st.muon_step(0.02, 0.95, 0.0)
    st.check()
    for tid, (pname, *_r) in enumerate(specs):
        if pname in V0:
            assert np.array_equal(f64(st.get(tid, g.KIND_NORMUON_V)), V0[pname].astype(np.float32))
    # reset the momentum and weights, then one NorMuon step from the preset V
    for tid, (pname, r, c, grp) in enumerate(specs):
        if pname in V0:
            st.set(tid, params[pname])
            st.set(tid, np.zeros((r, c)), kind=g.KIND_MOM)
    st.muon_step_normuon(0.02, 0.95, 0.0, 0.5)
    st.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        if pname not in V0:
            continue
        W0 = params[pname].astype(np.float64)
        V0f = V0[pname].astype(np.float32).astype(np.float64)
        W_ref, _, V_ref = oo.muon_step(W0, G[pname], np.zeros((r, c)), 0.02, 0.95, 0.0, normuon_V=V0f,
                                       normuon_beta2=0.5)
        assert relfro(f64(st.get(tid, g.KIND_PARAM)) - W0, W_ref - W0) <= MUON_RELFRO, pname
        assert relfro(f64(st.get(tid, g.KIND_NORMUON_V)), V_ref) <= 2 * MUON_RELFRO, pname


def test_normuon_rejects_bad_beta2(torch):
    import gpt_pretraining_step_b200 as g
    st = build(torch, SMALL["tiny"])
    for b in (1.0, -0.1, float("nan")):
        with pytest.raises(g.GptError):
            st.muon_step_normuon(0.02, 0.95, 0.0, b)


@pytest.mark.parametrize("normuon_beta2", [-1.0, 0.9])
def test_muon_by_layer_ranges_equals_whole_model(torch, normuon_beta2):
    """The ranges of a sharded optimizer step (layers 0-1, 2, 3) give bit for
    bit the whole-model Muon / NorMuon update, and the block regions address
    the tensors gpt_get_tensor returns."""
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=4, d_model=256, vocab=1000, batch=2, seq_len=64)
    params = syn.init_params(s, seed=31)
    specs = syn.param_specs(s)
    a, b = build(torch, s, params), build(torch, s, params)
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp == "muon":
            G = syn.gaussian((r, c), seed=500 + tid)
            a.set(tid, G, kind=g.KIND_GRAD)
            b.set(tid, G, kind=g.KIND_GRAD)
    for _ in range(2):
        if normuon_beta2 < 0:
            a.muon_step(0.02, 0.95, 0.01)
        else:
            a.muon_step_normuon(0.02, 0.95, 0.01, normuon_beta2)
        for l0, l1 in ((0, 2), (2, 3), (3, 3), (3, 4)):
            b.muon_step_layers(l0, l1, 0.02, 0.95, 0.01, normuon_beta2)
    a.check()
    b.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp != "muon":
            continue
        for kind in (g.KIND_PARAM, g.KIND_MOM) + ((g.KIND_NORMUON_V,) if normuon_beta2 >= 0 else ()):
            assert torch.equal(a.get(tid, kind), b.get(tid, kind)), (pname, kind)
    for kind in range(4):
        assert torch.equal(a.block_region(g.REGION_BF16, kind, 0, 4), b.block_region(g.REGION_BF16, kind, 0, 4))
        l, (pname, r, c, _) = 2, specs[2 + 4 * 2 + kind]
        master = b.block_region(g.REGION_MASTER, kind, l, l + 1).view(r, c)
        assert torch.equal(master, b.get(2 + 4 * l + kind, g.KIND_PARAM))
        assert torch.equal(b.block_region(g.REGION_BF16, kind, l, l + 1).view(r, c), master.to(torch.bfloat16))
        assert torch.equal(b.block_region(g.REGION_GRAD, kind, l, l + 1).view(r, c),
                           b.get(2 + 4 * l + kind, g.KIND_GRAD))
    with pytest.raises(g.GptError):
        b.muon_step_layers(3, 5)


def test_adamw_step_matches_oracle(torch):
    import gpt_pretraining_step_b200 as g
    s = SMALL["ragged"]
    params = syn.init_params(s, seed=3)
    st = build(torch, s, params)
    m = {0: np.zeros((s.vocab, s.d_model)), 1: np.zeros((s.d_model, s.vocab))}
    v = {k_: np.zeros_like(a) for k_, a in m.items()}
    p = {0: params["wte"].astype(np.float64), 1: params["lm_head"].astype(np.float64)}
    for step in (1, 2, 3):
        for tid in (0, 1):
            grad = syn.gaussian(p[tid].shape, seed=10 * step + tid, std=1e-3)
            st.set(tid, grad, kind=g.KIND_GRAD)
            p[tid], m[tid], v[tid] = oo.adamw_step(p[tid], grad, m[tid], v[tid], step, lr=3e-3, beta1=0.8,
                                                   beta2=0.95, eps=1e-10, weight_decay=0.1)
        st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.1)
        st.check()
        for tid in (0, 1):
            got = f64(st.get(tid, g.KIND_PARAM))
            assert np.abs(got - p[tid]).max() < 1e-6, (step, tid)


@pytest.mark.parametrize("ns_tf32_steps", [-1, 3, 5])
def test_whole_step_matches_oracle(torch, ns_tf32_steps):
    import gpt_pretraining_step_b200 as g
    s = SMALL["tiny"]
    params = syn.init_params(s, seed=4)
    tok, tgt = syn.tokens(s, seed=5), syn.targets(s, seed=6)
    st = build(torch, s, params, ns_tf32_steps=ns_tf32_steps)
    hp = g.HParams(muon_lr=0.02, muon_momentum=0.95, muon_wd=0.0, adam_lr=3e-3, adam_beta1=0.8, adam_beta2=0.95,
                   adam_eps=1e-10, adam_wd=0.0)
    st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda())
    st.check()
    ggpu = {pname: f64(st.get(tid, g.KIND_GRAD)) for tid, (pname, *_r) in enumerate(syn.param_specs(s))}
    loss = st.train_step_host(tok.astype(np.int32), tgt.astype(np.int32), hp)
    loss_ref, grads, _ = om.fwd_bwd(params, tok, tgt, s.depth)

    assert abs(loss - loss_ref) / loss_ref <= LOSS_RTOL
    for tid, (pname, r, c, grp) in enumerate(syn.param_specs(s)):
        W0 = params[pname].astype(np.float64)
        if grp == "muon":
            W_ref, _ = oo.muon_step(W0, grads[pname], np.zeros((r, c)), 0.02, 0.95, 0.0)
        else:
            W_ref, _, _ = oo.adamw_step(W0, grads[pname], np.zeros((r, c)), np.zeros((r, c)), 1, 3e-3, 0.8, 0.95,
                                        1e-10, 0.0)
        W_got = f64(st.get(tid, g.KIND_PARAM))
        if grp == "muon":
            # the update inherits the bf16 gradient error, amplified by Newton-Schulz
            eg = relfro(ggpu[pname], grads[pname])
            kappa = ns_amplification(grads[pname])
            err = relfro(W_got - W0, W_ref - W0)
            assert err <= MUON_RELFRO + 1.5 * kappa * eg, (pname, err, kappa, eg)
        else:
            # step 1 of AdamW is lr * sign(g) wherever |g| >> eps: compare where the sign is well defined
            gg = grads[pname]
            sure = np.abs(gg) > 1e-2 * np.abs(gg).max()
            agree = np.mean(np.sign((W_got - W0)[sure]) == np.sign((W_ref - W0)[sure]))
            assert agree >= 0.999, (pname, agree)


def ns_amplification(G, rel=1e-2, trials=3, seed=0):
    """Relative change of NS(G) per relative change of G, for random perturbations (oracle only)."""
    rng = np.random.default_rng(seed)
    base = oo.newton_schulz(G)
    worst = 0.0
    for _ in range(trials):
        d = rng.standard_normal(G.shape)
        d *= rel * np.linalg.norm(G) / np.linalg.norm(d)
        worst = max(worst, relfro(oo.newton_schulz(G + d), base) / rel)
    return worst


@pytest.mark.parametrize("name", list(SMALL))
def test_muon_on_model_gradients(torch, name):
    # Newton-Schulz precision on the spectra real gradients have: the oracle's
    # gradients of the seeded model are the (identical) input of both sides
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=7)
    tok, tgt = syn.tokens(s, seed=8), syn.targets(s, seed=9)
    _, grads, _ = om.fwd_bwd(params, tok, tgt, s.depth)
    st = build(torch, s, params)
    specs = syn.param_specs(s)
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp == "muon":
            st.set(tid, grads[pname].astype(np.float32), kind=g.KIND_GRAD)
    st.muon_step(0.02, 0.95, 0.0)
    st.check()
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp != "muon":
            continue
        G32 = grads[pname].astype(np.float32).astype(np.float64)
        W0 = params[pname].astype(np.float64)
        W_ref, _ = oo.muon_step(W0, G32, np.zeros((r, c)), 0.02, 0.95, 0.0)
        err = relfro(f64(st.get(tid, g.KIND_PARAM)) - W0, W_ref - W0)
        assert err <= MUON_RELFRO, (pname, err)


# ------------------------------------------------- full size (bench launch shape)

@pytest.fixture(scope="module")
def d20(torch):
    s = syn.config_shape("d20")
    params = syn.init_params(s, seed=0)
    st = build(torch, s, params)
    tok, tgt = syn.tokens(s), syn.targets(s)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    return s, params, st, tok, tgt, loss


def test_d20_loss_matches_gaussian_closed_form(d20):
    s, params, st, tok, tgt, loss = d20
    sig2 = 0.02 ** 2 * s.d_model
    expect = math.log(s.vocab) + sig2 / 2 - (math.exp(sig2) - 1) / (2 * s.vocab)
    assert abs(loss - expect) < 4 * math.sqrt(sig2 / s.tokens) + 1e-3


def test_d20_prefix_losses_match_oracle(d20):
    # causality: the losses of the first P positions of sequence 0 depend only on
    # its first P tokens, so the oracle can compute them alone
    s, params, st, tok, tgt, loss = d20
    P = 128
    got = f64(st.row_loss())[0, :P]
    _, cache = om.forward(params, tok[:1, :P], tgt[:1, :P], s.depth)
    ref = cache["row_loss"]
    assert np.abs(got - ref).max() / np.abs(ref).mean() <= LOSS_RTOL
    assert abs(got.mean() - ref.mean()) / ref.mean() <= 1e-3


def test_d20_embedding_gradient_rows(d20, torch):
    import gpt_pretraining_step_b200 as g
    s, params, st, tok, tgt, loss = d20
    E = st.get(0, g.KIND_GRAD)
    nz = torch.nonzero(E.abs().sum(dim=1) > 0).flatten().cpu().numpy()
    assert set(nz.tolist()) == set(np.unique(tok).tolist())


def test_d20_muon_sampled_matrices(d20, torch):
    import gpt_pretraining_step_b200 as g
    s, params, st, tok, tgt, loss = d20
    specs = syn.param_specs(s)
    Gs = {}
    for tid, (pname, r, c, grp) in enumerate(specs):
        if grp == "muon":
            Gs[tid] = syn.gaussian((r, c), seed=1000 + tid)
            st.set(tid, Gs[tid], kind=g.KIND_GRAD)
            st.set(tid, np.zeros((r, c), np.float32), kind=g.KIND_MOM)
    W0 = {tid: f64(st.get(tid, g.KIND_PARAM)) for tid in Gs}
    st.muon_step(0.02, 0.95, 0.0)
    st.check()
    for tid in (2, 2 + 4 * 7 + 1, 2 + 4 * 13 + 2, 2 + 4 * 19 + 3):
        W_ref, _ = oo.muon_step(W0[tid], Gs[tid], np.zeros_like(W0[tid]), 0.02, 0.95, 0.0)
        W_got = f64(st.get(tid, g.KIND_PARAM))
        assert relfro(W_got - W0[tid], W_ref - W0[tid]) <= MUON_RELFRO, specs[tid][0]


# ----------------------------------------------------------------- fp8 e4m3

FP8_LOSS_RTOL = 3e-2
FP8_GRAD_COS = 0.99


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_step_matches_oracle(torch, name):
    # the four block projections of the forward on e4m3 operands with dynamic
    # per-tensor scales, against the fp64 oracle at the fp8 tolerances
    import gpt_pretraining_step_b200 as g
    s = SMALL[name]
    params = syn.init_params(s, seed=0)
    tok, tgt = syn.tokens(s), syn.targets(s)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model, precision=1)
    for tid, (pname, *_r) in enumerate(syn.param_specs(s)):
        st.set(tid, params[pname])
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.check()
    loss_ref, grads, _ = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= FP8_LOSS_RTOL
    for tid, (pname, *_r) in enumerate(syn.param_specs(s)):
        c = cosine(f64(st.get(tid, g.KIND_GRAD)), grads[pname])
        assert c >= FP8_GRAD_COS, (pname, c)
    st.muon_step(0.02, 0.95, 0.0)
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()


def test_d26_fp8_initial_loss(torch):
    # the d26 configuration with fp8 projections: the initial loss keeps the
    # Gaussian closed form within the fp8 tolerance
    import gpt_pretraining_step_b200 as g
    s = syn.config_shape("d26")
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, precision=1)
    tok, tgt = syn.tokens(s), syn.targets(s)
    loss = float(st.fwd_bwd(torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()).item())
    st.muon_step(0.02, 0.95, 0.0)
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()
    sig2 = 0.02 ** 2 * s.d_model
    expect = math.log(s.vocab) + sig2 / 2 - (math.exp(sig2) - 1) / (2 * s.vocab)
    assert abs(loss - expect) / expect <= FP8_LOSS_RTOL
