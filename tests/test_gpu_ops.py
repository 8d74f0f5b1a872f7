"""Op-level parity of the CUDA kernels against the fp64 oracle (B200 only).

Each case uses seeded inputs with ragged sizes that span several tiles.
Tolerances follow from the arithmetic: bf16 operands are exact in fp64,
products accumulate in fp32 (relative error ~1e-6 per add), so GEMMs must
agree to ~1e-5 relative; attention rounds P to bf16 before P.V (relative
2^-9 per weight), so outputs agree to ~1e-2 relative; Newton-Schulz must
meet the 2e-2 relative Frobenius bound of the Muon update.
"""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as om
from oracle import optim as oo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as t
    import gpt_pretraining_step_b200 as g
    g.lib()
    return t


def bf16_t(torch, a):
    return torch.tensor(syn.round_to_bf16(np.asarray(a, dtype=np.float32))).to(torch.bfloat16).cuda()


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def relfro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cosine(a, b):
    a, b = a.ravel(), b.ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


@pytest.mark.parametrize("a_trans", [0, 1])
@pytest.mark.parametrize("b_trans", [0, 1])
@pytest.mark.parametrize("M,N,K,batch", [(264, 392, 200, 2), (128, 256, 64, 1), (8, 8, 8, 1), (520, 1032, 1000, 1)])
def test_matmul_bf16(torch, a_trans, b_trans, M, N, K, batch):
    import gpt_pretraining_step_b200 as g
    A = syn.round_to_bf16(syn.gaussian((batch, M, K), seed=M + K))
    B = syn.round_to_bf16(syn.gaussian((batch, K, N), seed=N + K + 1))
    At = A.transpose(0, 2, 1).copy() if a_trans else A
    Bt = B.transpose(0, 2, 1).copy() if b_trans else B
    C = g.matmul_bf16(bf16_t(torch, At), bf16_t(torch, Bt), M, N, K, batch=batch, a_trans=a_trans, b_trans=b_trans)
    torch.cuda.synchronize()
    ref = np.matmul(A.astype(np.float64), B.astype(np.float64))
    got = f64(C)
    assert relfro(got, ref) < 1e-5
    assert np.abs(got - ref).max() < 1e-4 * np.sqrt(K) * 4


def _tf32(a):
    # keep the 10 explicit mantissa bits the tensor cores read (truncation)
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


@pytest.mark.parametrize("b_trans", [1])
@pytest.mark.parametrize("M,N,K", [(128, 128, 32), (256, 384, 200), (136, 264, 136)])
def test_matmul_tf32(torch, b_trans, M, N, K):
    import gpt_pretraining_step_b200 as g
    A = syn.gaussian((M, K), seed=M + 3 * K)
    B = syn.gaussian((K, N), seed=N + 5 * K)
    Bs = B.T.copy() if b_trans else B
    C = g.matmul_tf32(torch.tensor(A).cuda(), torch.tensor(Bs).cuda(), M, N, K, b_trans=b_trans)
    torch.cuda.synchronize()
    got = f64(C)
    ref = _tf32(A) @ _tf32(B)
    err = relfro(got, ref)
    if err > 1e-4:
        exact = A.astype(np.float64) @ B.astype(np.float64)
        print("tf32 mismatch", b_trans, M, N, K, err, "vs exact", relfro(got, exact),
              "got[:2,:4]", got[:2, :4], "ref[:2,:4]", ref[:2, :4])
    assert err < 1e-4


def test_rmsnorm_fwd(torch):
    import gpt_pretraining_step_b200 as g
    x = syn.gaussian((300, 1280), seed=3, std=2.0)
    y, r = g.rmsnorm_fwd(torch.tensor(x).cuda())
    torch.cuda.synchronize()
    yr, rr = om.rms_norm(x.astype(np.float64))
    assert np.abs(f64(y) - yr).max() <= np.abs(yr).max() * 2 ** -8
    assert np.allclose(f64(r), rr[:, 0], rtol=1e-5)


def _attn_inputs(B, H, T, seed):
    # q, k as the QK-norm produces them (RMS 1 per head), v unit Gaussian
    q = syn.gaussian((B, H, T, 128), seed=seed)
    k = syn.gaussian((B, H, T, 128), seed=seed + 1)
    v = syn.gaussian((B, H, T, 128), seed=seed + 2)
    q = syn.round_to_bf16(om.rms_norm(q.astype(np.float64))[0].astype(np.float32))
    k = syn.round_to_bf16(om.rms_norm(k.astype(np.float64))[0].astype(np.float32))
    v = syn.round_to_bf16(v)
    return q, k, v


@pytest.mark.parametrize("B,H,T", [(2, 3, 200), (1, 1, 1), (1, 2, 64), (1, 1, 384), (2, 1, 129),
                                   (1, 2, 640), (2, 1, 1100), (1, 1, 1537)])
def test_attention_fwd(torch, B, H, T):
    import gpt_pretraining_step_b200 as g
    q, k, v = _attn_inputs(B, H, T, seed=T)
    o, lse = g.attention_fwd(bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v))
    torch.cuda.synchronize()
    ref, P = om.causal_attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64))
    got = f64(o).transpose(0, 2, 1, 3)           # [B, T, H, hd] -> [B, H, T, hd]
    assert relfro(got, ref) < 1e-2
    assert np.abs(got - ref).max() < 3e-2
    s = np.matmul(q.astype(np.float64), np.swapaxes(k.astype(np.float64), -1, -2)) / np.sqrt(128)
    s = np.where(np.triu(np.ones((T, T), bool), 1), -np.inf, s)
    lse_ref = om.logsumexp(s)
    assert np.abs(f64(lse) - lse_ref).max() < 2e-3


@pytest.mark.parametrize("B,H,T", [(2, 3, 200), (1, 1, 1), (1, 2, 256), (1, 1, 333), (1, 2, 640), (2, 1, 1100)])
def test_attention_bwd(torch, B, H, T):
    import gpt_pretraining_step_b200 as g
    q, k, v = _attn_inputs(B, H, T, seed=7 * T)
    dout = syn.round_to_bf16(syn.gaussian((B, T, H, 128), seed=T + 99))
    qt, kt, vt = bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v)
    o, lse = g.attention_fwd(qt, kt, vt)
    dq, dk, dv = g.attention_bwd(qt, kt, vt, o, lse, bf16_t(torch, dout))
    torch.cuda.synchronize()
    _, P = om.causal_attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64))
    dq_r, dk_r, dv_r = om.causal_attention_bwd(dout.astype(np.float64).transpose(0, 2, 1, 3),
                                               q.astype(np.float64), k.astype(np.float64),
                                               v.astype(np.float64), P)
    for got, ref in ((f64(dq), dq_r), (f64(dk), dk_r), (f64(dv), dv_r)):
        if np.linalg.norm(ref) < 1e-9:
            # T = 1: the softmax is constant, so dq = dk = 0 exactly
            assert np.abs(got).max() < 1e-6
            continue
        assert cosine(got, ref) > 0.9999
        assert relfro(got, ref) < 2e-2


# grouped kv heads and sliding windows: windows below, at and across tile
# edges, a window of 0 (each query sees itself), one wider than the row
VARIANTS = [(2, 4, 2, 333, 100), (1, 3, 1, 520, 0), (1, 2, 2, 700, 128), (1, 4, 4, 1000, 255),
            (2, 2, 1, 200, 1000), (1, 6, 3, 1024, 127), (1, 2, 1, 900, 129)]


def _kv_inputs(B, H, Hkv, T, seed):
    q, k, v = _attn_inputs(B, H, T, seed)
    return q, k[:, :Hkv].copy(), v[:, :Hkv].copy()


@pytest.mark.parametrize("B,H,Hkv,T,window", VARIANTS)
def test_attention_fwd_window_gqa(torch, B, H, Hkv, T, window):
    import gpt_pretraining_step_b200 as g
    q, k, v = _kv_inputs(B, H, Hkv, T, seed=T + window)
    o, lse = g.attention_fwd(bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v), window=window)
    torch.cuda.synchronize()
    ref, _ = om.attention(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), window=window)
    got = f64(o).transpose(0, 2, 1, 3)
    assert relfro(got, ref) < 1e-2
    assert np.abs(got - ref).max() < 3e-2
    kq = om.kv_for_queries(k.astype(np.float64), H)
    s = np.matmul(q.astype(np.float64), np.swapaxes(kq, -1, -2)) / np.sqrt(128)
    s = np.where(om.attention_hidden(T, window), -np.inf, s)
    assert np.abs(f64(lse) - om.logsumexp(s)).max() < 2e-3


@pytest.mark.parametrize("B,H,Hkv,T,window", VARIANTS)
def test_attention_bwd_window_gqa(torch, B, H, Hkv, T, window):
    import gpt_pretraining_step_b200 as g
    q, k, v = _kv_inputs(B, H, Hkv, T, seed=3 * T + window)
    dout = syn.round_to_bf16(syn.gaussian((B, T, H, 128), seed=T + window + 5))
    qt, kt, vt = bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v)
    o, lse = g.attention_fwd(qt, kt, vt, window=window)
    dq, dk, dv = g.attention_bwd(qt, kt, vt, o, lse, bf16_t(torch, dout), window=window)
    torch.cuda.synchronize()
    q64, k64, v64 = q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)
    _, P = om.attention(q64, k64, v64, window=window)
    refs = om.attention_bwd(dout.astype(np.float64).transpose(0, 2, 1, 3), q64, k64, v64, P)
    assert f64(dk).shape == k.shape and f64(dv).shape == v.shape
    for name, got, ref in zip("q k v".split(), (f64(dq), f64(dk), f64(dv)), refs):
        if window == 0 and name in "qk":
            # one visible key per query: the softmax is constant, dq = dk = 0
            assert np.abs(got).max() < 1e-4, name
            continue
        assert cosine(got, ref) > 0.9999, name
        assert relfro(got, ref) < 2e-2, name


@pytest.mark.parametrize("Hkv,window", [(10, 1024), (2, -1), (5, 512)])
def test_attention_variants_at_d20_shape_sampled(torch, Hkv, window):
    """The d20 attention shape (B 16, H 10, T 2048) with grouped kv heads and
    windows, checked on sampled heads: o, lse and dq of two query heads, dk
    and dv of one kv head (the sum over its whole group)."""
    import gpt_pretraining_step_b200 as g
    B, H, T = 16, 10, 2048
    G = H // Hkv
    q, k, v = _kv_inputs(B, H, Hkv, T, seed=Hkv + 7)
    dout = syn.round_to_bf16(syn.gaussian((B, T, H, 128), seed=Hkv + 9))
    qt, kt, vt = bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v)
    o, lse = g.attention_fwd(qt, kt, vt, window=window)
    dq, dk, dv = g.attention_bwd(qt, kt, vt, o, lse, bf16_t(torch, dout), window=window)
    torch.cuda.synchronize()
    w = None if window < 0 else window
    for b, hk in ((3, 0), (12, Hkv - 1)):
        heads = list(range(hk * G, hk * G + G))
        q64 = q[b:b + 1, heads].astype(np.float64)
        k64, v64 = k[b:b + 1, hk:hk + 1].astype(np.float64), v[b:b + 1, hk:hk + 1].astype(np.float64)
        ref, P = om.attention(q64, k64, v64, window=w)
        got_o = f64(o[b, :, heads]).transpose(1, 0, 2)[None]
        assert relfro(got_o, ref) < 1e-2, (b, hk)
        dy = dout[b:b + 1, :, heads].astype(np.float64).transpose(0, 2, 1, 3)
        dq_r, dk_r, dv_r = om.attention_bwd(dy, q64, k64, v64, P)
        for got, r in ((f64(dq[b, heads])[None], dq_r), (f64(dk[b, hk])[None, None], dk_r),
                       (f64(dv[b, hk])[None, None], dv_r)):
            assert cosine(got, r) > 0.9999 and relfro(got, r) < 2e-2, (b, hk)


def test_attention_rejects_bad_head_split(torch):
    import gpt_pretraining_step_b200 as g
    q, k, v = _kv_inputs(1, 3, 2, 64, seed=1)
    with pytest.raises(g.GptError):
        g.attention_fwd(bf16_t(torch, q), bf16_t(torch, k), bf16_t(torch, v))


@pytest.mark.parametrize("batch,rows,cols", [(2, 256, 768), (1, 640, 128), (3, 128, 128), (1, 136, 264),
                                              (1, 600, 704), (2, 520, 1032)])
@pytest.mark.parametrize("tf32_steps", [-1, 0, 3, 5])
def test_newton_schulz(torch, batch, rows, cols, tf32_steps):
    import gpt_pretraining_step_b200 as g
    G = syn.gaussian((batch, rows, cols), seed=rows + cols)
    X = g.newton_schulz(torch.tensor(G).cuda(), tf32_steps=tf32_steps)
    torch.cuda.synchronize()
    got = f64(X)
    for z in range(batch):
        ref = oo.newton_schulz(G[z].astype(np.float64))
        err = relfro(got[z], ref)
        assert err < (1e-2 if tf32_steps in (-1, 5) else 2e-2), (z, err)


def test_quantize_e4m3_bit_exact(torch):
    # the scale 448 / amax and the product x * scale are formed in fp32 on both
    # sides (the decision precision of the kernel); the rounding to the e4m3 grid
    # is the oracle's
    import gpt_pretraining_step_b200 as g
    from oracle import fp8 as of
    x = syn.round_to_bf16(np.concatenate([syn.gaussian(40000, seed=21) * 3.0,
                                          syn.gaussian(1000, seed=22) * 1e-3, [0.0, -7.5]]).astype(np.float32))
    q, inv = g.quantize_e4m3(bf16_t(torch, x))
    torch.cuda.synchronize()
    amax = np.float32(np.abs(x).max())
    sc = np.float32(448.0) / amax
    want = of.round_e4m3((x * sc).astype(np.float32).astype(np.float64))
    got = q.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)
    assert np.array_equal(got, want)
    assert float(inv.item()) == float(amax / np.float32(448.0))


@pytest.mark.parametrize("b_trans", [0, 1])
@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (200, 272, 160)])
def test_matmul_fp8(torch, b_trans, M, N, K):
    import gpt_pretraining_step_b200 as g
    from oracle import fp8 as of
    qa = of.round_e4m3(syn.gaussian((M, K), seed=M + K) * 100)
    qb = of.round_e4m3(syn.gaussian((K, N), seed=N + K) * 100)
    ta = torch.tensor(qa, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
    bs = qb.T.copy() if b_trans else qb
    tb = torch.tensor(bs, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).cuda()
    inv_a = torch.tensor([0.5], dtype=torch.float32).cuda()
    inv_b = torch.tensor([0.125], dtype=torch.float32).cuda()
    C = g.matmul_fp8(ta, tb, M, N, K, inv_a, inv_b, b_trans=bool(b_trans))
    torch.cuda.synchronize()
    ref = (qa @ qb) * 0.5 * 0.125
    assert relfro(f64(C), ref) < 1e-6


@pytest.mark.parametrize("stream", ["zipf", "uniform"])
def test_embedding_bwd_at_benchmark_size(torch, stream):
    """The embedding gradient at the benchmark's 32768 positions and width
    1280: a Zipf(1.1) id stream (the skew of natural text: thousands of
    positions on the first ids) and a uniform one, against the oracle's
    scatter.  A row that occurs once is an exact copy; rows are summed in
    fp32, so a row of n positions agrees to a few ulps of its magnitude
    sum; the result is deterministic and accumulate adds onto the output."""
    import gpt_pretraining_step_b200 as g
    s = syn.make_shape(depth=20, batch=16, seq_len=2048)
    tok = (syn.zipf_tokens(s, seed=3) if stream == "zipf" else syn.tokens(s, seed=1)).reshape(-1)
    dx = syn.gaussian((s.tokens, s.d_model), seed=31)
    ref = om.embedding_bwd(tok, dx.astype(np.float64), s.vocab)
    mag = om.embedding_bwd(tok, np.abs(dx).astype(np.float64), s.vocab)
    t_tok = torch.tensor(tok).cuda()
    t_dx = torch.tensor(dx).cuda()
    got = g.embedding_bwd(t_tok, t_dx, s.vocab)
    again = g.embedding_bwd(t_tok, t_dx, s.vocab)
    torch.cuda.synchronize()
    assert torch.equal(got, again)
    counts = np.bincount(tok, minlength=s.vocab)
    if stream == "zipf":
        assert counts.max() > 2000
    G = f64(got)
    assert np.all(G[counts == 0] == 0.0)
    once = counts == 1
    assert np.array_equal(G[once], ref[once])
    assert np.all(np.abs(G - ref) <= 1e-6 * mag + 1e-30)
    twice = g.embedding_bwd(t_tok, t_dx, s.vocab, dwte=got.clone(), accumulate=True)
    torch.cuda.synchronize()
    assert np.all(np.abs(f64(twice) - 2 * ref) <= 2e-6 * mag + 1e-30)
