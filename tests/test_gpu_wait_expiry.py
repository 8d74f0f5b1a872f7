"""Failure detection on the GPU: bounded device waits that run out (B200 only).

Every wait inside the GEMM and attention kernels (TMA loads landing, tensor
core products completing, the softmax warps handing tiles over) gives up
after a bound of SM cycles; the kernel then lets its in-flight copies land,
frees its tensor memory, returns, and the error is latched in a device word
that gpt_check (a context) or gpt_op_check (the op-level calls) reports.
These tests shorten the bound to a few hundred cycles, far below a TMA
load's latency, so the waits of ordinary launches expire; they check that
the expiry is reported as GPT_ETIMEOUT, and that with the default bound
restored the same context and the same op-level calls give oracle-matching
results again (the GPU was left usable).  No fault, trap or hang is
involved: every wait stays bounded.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as om

pytestmark = pytest.mark.gpu

SHORT = 300   # SM cycles


@pytest.fixture(scope="module")
def torch():
    import torch as t
    import gpt_pretraining_step_b200 as g
    g.lib()
    g.op_set_wait_limit(0)
    try:
        g.op_check()
    except g.GptError:
        pass
    return t


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def cosine(a, b):
    a, b = np.ravel(a), np.ravel(b)
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def _expect_timeout(g, fn):
    import gpt_pretraining_step_b200 as gg
    with pytest.raises(gg.GptError) as e:
        fn()
    assert e.value.code == g.GPT_ETIMEOUT, str(e.value)


def test_op_level_expiry_is_reported_and_calls_recover(torch):
    import gpt_pretraining_step_b200 as g
    M, N, K = 1024, 768, 2048
    A = syn.round_to_bf16(syn.gaussian((M, K), seed=61))
    Bm = syn.round_to_bf16(syn.gaussian((K, N), seed=62))
    tA = torch.tensor(A).to(torch.bfloat16).cuda()
    tB = torch.tensor(Bm).to(torch.bfloat16).cuda()
    B_, H, T = 1, 2, 512
    q, k, v = (torch.tensor(syn.round_to_bf16(syn.gaussian((B_, H, T, 128), seed=70 + i))).to(torch.bfloat16).cuda()
               for i in range(3))
    do = torch.tensor(syn.round_to_bf16(syn.gaussian((B_, T, H, 128), seed=73))).to(torch.bfloat16).cuda()
    G = torch.tensor(syn.gaussian((2, 256, 512), seed=74)).cuda()
    g.op_set_wait_limit(SHORT)
    try:
        g.matmul_bf16(tA, tB, M, N, K)
        _expect_timeout(g, g.op_check)
        o, lse = g.attention_fwd(q, k, v)
        _expect_timeout(g, g.op_check)
        g.attention_bwd(q, k, v, o, lse, do)
        _expect_timeout(g, g.op_check)
        g.newton_schulz_noalloc(G)
        _expect_timeout(g, g.op_check)
    finally:
        g.op_set_wait_limit(0)
    # the default bound again: the same calls agree with the oracle
    C = g.matmul_bf16(tA, tB, M, N, K)
    o, lse = g.attention_fwd(q, k, v)
    g.op_check()
    ref = A.astype(np.float64) @ Bm.astype(np.float64)
    got = f64(C)[0]
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-5
    y, _ = om.causal_attention(*(f64(t) for t in (q, k, v)))
    assert np.abs(f64(o) - y.transpose(0, 2, 1, 3)).max() < 2e-2
    # a clean check reports nothing
    g.op_check()


def test_context_expiry_is_reported_and_context_survives(torch):
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=2, d_model=256, vocab=1000, batch=2, seq_len=200)
    params = syn.init_params(s, seed=81)
    tok, tgt = syn.tokens(s, seed=82), syn.targets(s, seed=83)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model)
    for tid, (name, *_r) in enumerate(syn.param_specs(s)):
        st.set(tid, params[name])
    ttok, ttgt = torch.tensor(tok).cuda(), torch.tensor(tgt).cuda()
    st.set_wait_limit(SHORT)
    st.fwd_bwd(ttok, ttgt)
    _expect_timeout(g, st.check)
    st.set_wait_limit(0)
    loss = float(st.fwd_bwd(ttok, ttgt).item())
    st.check()
    loss_ref, grads, _ = om.fwd_bwd(params, tok, tgt, s.depth)
    assert abs(loss - loss_ref) / loss_ref <= 1e-2
    for tid, (pname, *_r) in enumerate(syn.param_specs(s)):
        c = cosine(f64(st.get(tid, g.KIND_GRAD)), grads[pname])
        assert c >= 0.999, (pname, c)
    st.muon_step(0.02, 0.95, 0.0)
    st.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    st.check()
