"""Pins of the fp64 model oracle against what the pages and mathematics fix (CPU only)."""
import numpy as np
import pytest

import synthetic as syn
from oracle import model as om


def small_case(depth=2, d=128, vocab=64, batch=2, seq=16, seed=0, std=0.02):
    s = syn.make_shape(depth=depth, batch=batch, seq_len=seq, vocab=vocab, d_model=d)
    p = syn.init_params(s, seed=seed, std=std)
    tok = syn.tokens(s, seed=seed + 1)
    tgt = syn.targets(s, seed=seed + 2)
    return s, p, tok, tgt


# --- loss closed forms ------------------------------------------------------

def test_zero_lm_head_loss_is_log_vocab():
    s, p, tok, tgt = small_case()
    p["lm_head"] = np.zeros_like(p["lm_head"])
    loss, _ = om.forward(p, tok, tgt, s.depth)
    assert loss == pytest.approx(np.log(s.vocab), abs=1e-12)


def test_zero_lm_head_grad_closed_form():
    # with z = 0, dz = (1/V - onehot(target)) / M, so every row of dW_lm sums to 0
    # and the target-column total is -(sum of xf rows with that target)/M*(1-1/V)
    s, p, tok, tgt = small_case()
    p["lm_head"] = np.zeros_like(p["lm_head"])
    loss, g, cache = om.fwd_bwd(p, tok, tgt, s.depth)
    assert np.abs(g["lm_head"].sum(axis=1)).max() < 1e-14
    xf = cache["xf"]
    M = s.tokens
    t = tgt.reshape(-1)
    expect = xf.sum(0)[:, None] / (M * s.vocab) * np.ones((1, s.vocab))
    for m in range(M):
        expect[:, t[m]] -= xf[m] / M
    assert np.allclose(g["lm_head"], expect, atol=1e-15)


def test_initial_loss_matches_gaussian_logit_closed_form():
    # xf has RMS 1 so, given xf, the logits are iid N(0, sigma^2) with
    # sigma^2 = std^2 * d; E[loss] = ln V + sigma^2/2 - (e^{sigma^2}-1)/(2V)
    s = syn.make_shape(depth=1, batch=4, seq_len=256, vocab=4096, d_model=256)
    p = syn.init_params(s, seed=5)
    tok, tgt = syn.tokens(s, seed=6), syn.targets(s, seed=7)
    loss, cache = om.forward(p, tok, tgt, s.depth)
    sig2 = 0.02 ** 2 * s.d_model
    expect = np.log(s.vocab) + sig2 / 2 - (np.exp(sig2) - 1) / (2 * s.vocab)
    # the target logit term dominates the sampling error: std ~ sigma / sqrt(M)
    assert abs(loss - expect) < 4 * np.sqrt(sig2 / s.tokens)
    # and the oracle's own logits have the variance the closed form assumes
    assert np.var(cache["z"]) == pytest.approx(sig2, rel=0.05)


def test_zero_blocks_are_identity():
    # with every block matrix zero the residual stream passes through unchanged,
    # so the loss equals that of the embedding -> norm -> lm_head model
    s, p, tok, tgt = small_case(depth=3)
    for name, *_ in syn.param_specs(s):
        if name.startswith("h"):
            p[name] = np.zeros_like(p[name])
    loss, _ = om.forward(p, tok, tgt, s.depth)
    loss0, _ = om.forward(p, tok, tgt, 0)
    assert loss == pytest.approx(loss0, abs=1e-13)


def test_single_position_attention_is_value():
    # T = 1: softmax over one key is 1, so attention returns v exactly
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((2, 3, 1, 128)) for _ in range(3))
    y, P = om.causal_attention(q, k, v)
    assert np.array_equal(P, np.ones_like(P))
    assert np.allclose(y, v, atol=0)


def test_attention_scale_and_mask():
    # two positions; q1.k0/sqrt(128) = 0 and q1.k1/sqrt(128) = ln 3 give
    # weights (1/4, 3/4) on row 1; row 0 sees only key 0
    hd = 128
    q = np.zeros((1, 1, 2, hd)); k = np.zeros((1, 1, 2, hd)); v = np.zeros((1, 1, 2, hd))
    q[..., 1, 0] = 1.0
    k[..., 1, 0] = np.log(3.0) * np.sqrt(hd)
    k[..., 0, 1] = 5.0           # orthogonal to q1
    q[..., 0, 1] = 7.0
    v[..., 0, 2] = 1.0
    v[..., 1, 3] = 1.0
    y, P = om.causal_attention(q, k, v)
    assert P[0, 0, 0].tolist() == [1.0, 0.0]
    assert np.allclose(P[0, 0, 1], [0.25, 0.75], atol=1e-15)
    assert np.allclose(y[0, 0, 1, 2:4], [0.25, 0.75], atol=1e-15)


def test_equal_keys_give_prefix_mean():
    rng = np.random.default_rng(4)
    T, hd = 9, 128
    q = rng.standard_normal((1, 1, T, hd))
    k = np.tile(rng.standard_normal((1, 1, 1, hd)), (1, 1, T, 1))
    v = rng.standard_normal((1, 1, T, hd))
    y, _ = om.causal_attention(q, k, v)
    prefix_mean = np.cumsum(v, axis=2) / np.arange(1, T + 1)[None, None, :, None]
    assert np.allclose(y, prefix_mean, atol=1e-13)


def test_causality():
    # changing tokens at positions > t leaves the per-position loss at <= t unchanged
    s, p, tok, tgt = small_case(seq=16)
    _, c1 = om.forward(p, tok, tgt, s.depth)
    tok2 = tok.copy()
    tok2[:, 10:] = (tok2[:, 10:] + 7) % s.vocab
    _, c2 = om.forward(p, tok2, tgt, s.depth)
    r1 = c1["row_loss"].reshape(s.batch, s.seq_len)
    r2 = c2["row_loss"].reshape(s.batch, s.seq_len)
    assert np.allclose(r1[:, :10], r2[:, :10], atol=1e-12, rtol=0)
    assert np.abs(r1[:, 10:] - r2[:, 10:]).max() > 1e-3


def test_target_index_moves_loss():
    s, p, tok, tgt = small_case()
    _, c1 = om.forward(p, tok, tgt, s.depth)
    tgt2 = tgt.copy()
    tgt2[0, 3] = (tgt2[0, 3] + 1) % s.vocab
    _, c2 = om.forward(p, tok, tgt2, s.depth)
    z = c1["z"]
    m = 3
    assert c2["row_loss"][m] - c1["row_loss"][m] == pytest.approx(
        z[m, tgt[0, 3]] - z[m, tgt2[0, 3]], abs=1e-12)


# --- RoPE / RMSNorm invariants -------------------------------------------------

def test_rope_is_rotation_and_relative():
    T, hd = 40, 128
    cos, sin = om.rope_angles(T, hd)
    rng = np.random.default_rng(1)
    q = rng.standard_normal(hd)
    k = rng.standard_normal(hd)
    Q = om.rope(np.tile(q, (T, 1)), cos, sin)
    K = om.rope(np.tile(k, (T, 1)), cos, sin)
    assert np.allclose(np.linalg.norm(Q, axis=1), np.linalg.norm(q), rtol=1e-14)
    dots = Q @ K.T
    for off in (0, 3, 17):
        diag = np.diagonal(dots, offset=off)
        assert np.allclose(diag, diag[0], atol=1e-11)
    # position 0 is the identity, and the backward is the inverse rotation
    assert np.allclose(Q[0], q, atol=0)
    assert np.allclose(om.rope_bwd(Q, cos, sin), np.tile(q, (T, 1)), atol=1e-13)


def test_rope_first_pair_angle():
    # pair 0 rotates by t radians (base^0 = 1); the last pair by t * base^(-126/128)
    cos, sin = om.rope_angles(8, 128)
    assert np.allclose(cos[:, 0], np.cos(np.arange(8)))
    assert np.allclose(sin[:, 63], np.sin(np.arange(8) * 10000.0 ** (-126 / 128)))


def test_rmsnorm_invariants():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 256)) * 3.0
    y, r = om.rms_norm(x)
    ms = np.mean(x * x, axis=1)
    assert np.allclose(np.mean(y * y, axis=1), ms / (ms + om.EPS), rtol=1e-14)
    y2, _ = om.rms_norm(10.0 * x)
    assert np.allclose(y, y2, atol=1e-7)   # scale invariant up to eps
    # gradient is orthogonal to y (scale invariance) up to the eps term
    dy = rng.standard_normal(x.shape)
    dx = om.rms_norm_bwd(dy, y, r)
    assert np.abs(np.sum(dx * x, axis=1)).max() < 1e-5


# --- finite differences --------------------------------------------------------

def _fd_check(p, tok, tgt, depth, names, n_coords=6, h=1e-5, seed=0, windows=None):
    loss, g, _ = om.fwd_bwd(p, tok, tgt, depth, windows=windows)
    rng = np.random.default_rng(seed)
    worst = 0.0
    for name in names:
        W = p[name].astype(np.float64)
        G = g[name]
        scale = np.abs(G).max()
        assert scale > 0, name
        if name == "wte":
            rows = np.unique(tok)
            coords = [(rng.choice(rows), rng.integers(W.shape[1])) for _ in range(n_coords)]
        else:
            # half at random, half at the largest gradient entries
            flat = np.argsort(np.abs(G).ravel())[-n_coords // 2:]
            coords = [np.unravel_index(i, W.shape) for i in flat]
            coords += [(rng.integers(W.shape[0]), rng.integers(W.shape[1]))
                       for _ in range(n_coords - len(coords))]
        for (i, j) in coords:
            pp = dict(p); Wp = W.copy(); Wp[i, j] += h; pp[name] = Wp
            lp, _ = om.forward(pp, tok, tgt, depth, keep=False, windows=windows)
            Wm = W.copy(); Wm[i, j] -= h; pp[name] = Wm
            lm, _ = om.forward(pp, tok, tgt, depth, keep=False, windows=windows)
            fd = (lp - lm) / (2 * h)
            err = abs(fd - G[i, j]) / scale
            worst = max(worst, err)
            assert err < 1e-6, (name, i, j, fd, G[i, j], scale)
    return worst


def test_finite_difference_every_tensor():
    s, p, tok, tgt = small_case(depth=2, d=128, vocab=64, batch=2, seq=16, std=0.05)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    names = [n for n, *_ in syn.param_specs(s)]
    _fd_check(p, tok, tgt, s.depth, names)


def test_finite_difference_two_heads():
    # two heads: checks the head split/merge and per-head QK norm
    s, p, tok, tgt = small_case(depth=1, d=256, vocab=48, batch=1, seq=12, std=0.05, seed=9)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    _fd_check(p, tok, tgt, s.depth, ["h0.c_qkv", "h0.c_proj", "wte"], n_coords=8)


def test_embedding_grad_rows():
    s, p, tok, tgt = small_case(vocab=64)
    _, g, _ = om.fwd_bwd(p, tok, tgt, s.depth)
    absent = np.setdiff1d(np.arange(s.vocab), np.unique(tok))
    assert len(absent) > 0
    assert np.all(g["wte"][absent] == 0.0)


def test_embedding_bwd_brute_force_with_repeated_tokens():
    # the gradient of a row copy, summed position by position in a plain loop;
    # a skewed id stream puts many positions on the same row
    rng = np.random.default_rng(7)
    tok = np.array([3, 3, 0, 5, 3, 5, 3, 9, 3, 0], dtype=np.int32)
    dx = rng.standard_normal((tok.size, 4))
    ref = np.zeros((10, 4))
    for m in range(tok.size):
        for c in range(4):
            ref[tok[m], c] += dx[m, c]
    got = om.embedding_bwd(tok, dx, 10)
    assert np.allclose(got, ref, rtol=0, atol=1e-14)
    assert np.all(got[[1, 2, 4, 6, 7, 8]] == 0.0)
    # a token on every position: the column sums
    assert np.allclose(om.embedding_bwd(np.full(10, 2), dx, 4)[2], dx.sum(axis=0), atol=1e-14)


def test_embedding_forward_is_row_copy():
    s, p, tok, tgt = small_case()
    # depth 0 and zero lm_head: xf = rms(wte[tok]); check via the cache
    _, c = om.forward(p, tok, tgt, 0)
    x0 = p["wte"][tok.reshape(-1)].astype(np.float64)
    xf, _ = om.rms_norm(x0)
    assert np.array_equal(c["xf"], xf)


# --- sliding window and grouped kv heads -------------------------------------
#
# Section "1. Modelo GPT" lists GQA (fewer kv heads than query heads) and
# sliding-window attention with a layer pattern such as "SSSL".  Reading: a
# window w lets query t see keys t - w .. t; query head h reads kv head
# h // (H / Hkv).

def _qkv(B, H, Hkv, T, hd, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, T, hd)), rng.standard_normal((B, Hkv, T, hd)),
            rng.standard_normal((B, Hkv, T, hd)))


def test_window_covering_the_row_is_causal():
    q, k, v = _qkv(2, 3, 3, 11, 16, 0)
    y0, p0 = om.causal_attention(q, k, v)
    for w in (10, 11, 50):
        y, p = om.attention(q, k, v, window=w)
        assert np.array_equal(y, y0) and np.array_equal(p, p0)


def test_window_zero_returns_own_value():
    q, k, v = _qkv(1, 4, 2, 7, 8, 1)
    y, p = om.attention(q, k, v, window=0)
    for h in range(4):
        assert np.array_equal(y[0, h], v[0, h // 2])
    assert np.array_equal(p[0, 0], np.eye(7))


def test_window_and_groups_brute_force():
    import math
    B, H, Hkv, T, hd, w = 2, 4, 2, 9, 8, 3
    q, k, v = _qkv(B, H, Hkv, T, hd, 2)
    y, _ = om.attention(q, k, v, window=w)
    for b in range(B):
        for h in range(H):
            g = h // (H // Hkv)
            for t in range(T):
                keys = list(range(max(0, t - w), t + 1))
                sc = [sum(q[b, h, t, i] * k[b, g, j, i] for i in range(hd)) / math.sqrt(hd) for j in keys]
                m = max(sc)
                e = [math.exp(x - m) for x in sc]
                z = sum(e)
                ref = [sum(e[n] / z * v[b, g, j, i] for n, j in enumerate(keys)) for i in range(hd)]
                assert np.allclose(y[b, h, t], ref, rtol=1e-12, atol=1e-12), (b, h, t)


def test_window_hides_keys_before_it():
    B, H, Hkv, T, hd, w = 1, 2, 1, 12, 8, 4
    q, k, v = _qkv(B, H, Hkv, T, hd, 3)
    y0, _ = om.attention(q, k, v, window=w)
    t = 9
    k2, v2 = k.copy(), v.copy()
    k2[:, :, : t - w] += 5.0
    v2[:, :, : t - w] -= 3.0
    y1, _ = om.attention(q, k2, v2, window=w)
    assert np.array_equal(y0[:, :, t:], y1[:, :, t:])
    assert not np.allclose(y0[:, :, t - 1], y1[:, :, t - 1])


def test_window_gqa_gradients_finite_difference():
    B, H, Hkv, T, hd, w = 1, 4, 2, 10, 8, 3
    q, k, v = _qkv(B, H, Hkv, T, hd, 4)
    R = np.random.default_rng(5).standard_normal((B, H, T, hd))
    y, p = om.attention(q, k, v, window=w)
    dq, dk, dv = om.attention_bwd(R, q, k, v, p)
    assert dk.shape == k.shape and dv.shape == v.shape
    rng = np.random.default_rng(6)
    h = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(rng.integers(n) for n in arr.shape)
            a = arr.copy()
            a[idx] += h
            args = {"q": q, "k": k, "v": v}
            args[name] = a
            lp = np.sum(om.attention(args["q"], args["k"], args["v"], window=w)[0] * R)
            a[idx] -= 2 * h
            lm = np.sum(om.attention(args["q"], args["k"], args["v"], window=w)[0] * R)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, np.abs(grad).max()), (name, idx, fd, grad[idx])


def test_layer_windows_pattern():
    assert om.layer_windows("SSSL", 64, 6) == [64, 64, 64, None, 64, 64]
    assert om.layer_windows("", 64, 3) == [None, None, None]
    assert om.layer_windows("L", 64, 2) == [None, None]
    with pytest.raises(ValueError):
        om.layer_windows("SXL", 64, 3)


def test_finite_difference_with_sliding_windows():
    s, p, tok, tgt = small_case(depth=2, d=128, vocab=48, batch=1, seq=14, std=0.05, seed=11)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    windows = om.layer_windows("SL", 3, s.depth)
    _fd_check(p, tok, tgt, s.depth, ["h0.c_qkv", "h1.c_qkv", "h0.c_proj"], n_coords=6, windows=windows)
    # the window changes the loss (layer 0 sees fewer keys)
    l0, _ = om.forward(p, tok, tgt, s.depth, keep=False)
    l1, _ = om.forward(p, tok, tgt, s.depth, keep=False, windows=windows)
    assert l0 != l1


# --- residual extras: per-layer residual / x0 scales and backout ---------------
#
# Section "1. Modelo GPT", efficiency tricks 1 and 3: x <- resid[i] x + x0l[i]
# x0 before block i, and x <- x - backout * x_mid after the last block, x_mid
# being the residual stream entering block L // 2.

def _extras_case(depth=2, seed=0, **kw):
    s, p, tok, tgt = small_case(depth=depth, seed=seed, **kw)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    return s, p, tok, tgt


def test_neutral_scalars_give_the_plain_model():
    s, p, tok, tgt = _extras_case(std=0.05)
    sc = np.zeros((1, 2 * s.depth + 26))
    sc[0, :s.depth] = 1.0
    l0, g0, _ = om.fwd_bwd(p, tok, tgt, s.depth)
    l1, g1, _ = om.fwd_bwd(dict(p, scalars=sc), tok, tgt, s.depth)
    assert l0 == l1
    for k in g0:
        assert np.array_equal(g0[k], g1[k]), k
    assert g1["scalars"].shape == (1, 2 * s.depth + 26)


def test_x0_only_inputs_reduce_to_the_last_block():
    # resid = 0, x0 scale = 1: every block reads the embedding, so only the
    # last block's contribution survives: a one-block model with its weights
    depth = 3
    s, p, tok, tgt = _extras_case(depth=depth, std=0.05, seed=4)
    sc = np.zeros((1, 2 * depth + 26))
    sc[0, depth:2 * depth] = 1.0
    loss, _ = om.forward(dict(p, scalars=sc), tok, tgt, depth, keep=False)
    one = {"wte": p["wte"], "lm_head": p["lm_head"]}
    for n in ("c_qkv", "c_proj", "c_fc", "mlp_proj"):
        one[f"h0.{n}"] = p[f"h{depth - 1}.{n}"]
    ref, _ = om.forward(one, tok, tgt, 1, keep=False)
    assert abs(loss - ref) < 1e-12


def test_backout_of_the_whole_stream_before_the_middle():
    # depth 2 with backout 1: the final stream is x_mid + f1(x_mid) - x_mid,
    # i.e. the last block's contribution alone on top of nothing
    s, p, tok, tgt = _extras_case(depth=2, std=0.05, seed=6)
    sc = np.zeros((1, 2 * 2 + 26))
    sc[0, :2] = 1.0
    sc[0, 4] = 1.0
    _, c = om.forward(dict(p, scalars=sc), tok, tgt, 2)
    _, cp = om.forward(p, tok, tgt, 2)
    # the stream entering block 1 is the final stream of block 0 alone
    _, c1 = om.forward({k: v for k, v in p.items() if not k.startswith("h1.")}, tok, tgt, 1)
    x_mid = c1["xf"] / c1["rf"]
    xf_ref, _ = om.rms_norm(cp["xf"] / cp["rf"] - x_mid)
    assert np.allclose(c["xf"], xf_ref, rtol=1e-9, atol=1e-12)


def test_finite_difference_with_residual_extras():
    s, p, tok, tgt = _extras_case(depth=2, std=0.05, seed=8, vocab=48, seq=12)
    p["scalars"] = syn.random_scalars(s, seed=9).astype(np.float64)
    names = [n for n, *_ in syn.param_specs(s, extras=True)]
    _fd_check(p, tok, tgt, s.depth, names, n_coords=4)


def test_smear_mixes_the_previous_embedding():
    # smear scale c with a zero gate weight vector: gate = c / 2, so the stream
    # entering block 0 is e[t] + (c / 2) e[t-1] (e[t] alone at t = 0)
    s, p, tok, tgt = _extras_case(depth=1, std=0.05, seed=12)
    sc = np.zeros((1, 2 + 26))
    sc[0, 0] = 1.0
    sc[0, 3] = 0.8
    _, c = om.forward(dict(p, scalars=sc), tok, tgt, 1)
    e = p["wte"][tok]                                    # [B, T, d]
    ref = e.copy()
    ref[:, 1:] += 0.4 * e[:, :-1]
    assert np.allclose(c["x0"].reshape(e.shape), ref, rtol=1e-12, atol=1e-15)
    # a token's smear never reaches across the sequence boundary
    assert np.array_equal(c["x0"].reshape(e.shape)[:, 0], e[:, 0])


# --- value embeddings ------------------------------------------------------------
#
# Section "1. Modelo GPT", value residual: on every other layer (from the
# first) v[t, h] += 3 sigmoid(xn1[t, :C] . W_g[:, h]) ve[tok[t], head h].

def _ve_case(depth=2, C=8, seed=0, **kw):
    s = syn.make_shape(depth=depth, batch=kw.pop("batch", 2), seq_len=kw.pop("seq", 10),
                       vocab=kw.pop("vocab", 40), d_model=kw.pop("d", 256))
    p = syn.init_params(s, seed=seed, std=0.05, ve_channels=C)
    rng = np.random.default_rng(seed + 1)
    p["ve_gate"] = rng.standard_normal(p["ve_gate"].shape).astype(np.float32) * 2.0
    p = {k: v.astype(np.float64) for k, v in p.items()}
    return s, p, syn.tokens(s, seed=seed + 2), syn.targets(s, seed=seed + 3)


def test_zero_value_embeddings_give_the_plain_model():
    s, p, tok, tgt = _ve_case()
    for l in syn.ve_layers(s.depth):
        p[f"ve{l}"] = np.zeros_like(p[f"ve{l}"])
    plain = {k: v for k, v in p.items() if not k.startswith("ve")}
    l0, g0, _ = om.fwd_bwd(plain, tok, tgt, s.depth)
    l1, g1, _ = om.fwd_bwd(p, tok, tgt, s.depth)
    assert l0 == l1
    for k in g0:
        assert np.array_equal(g0[k], g1[k]), k


def test_value_embedding_brute_force():
    import math
    s, p, tok, tgt = _ve_case(depth=1, C=4, batch=1, seq=5, d=256)
    _, c = om.forward(p, tok, tgt, 1)
    _, c0 = om.forward({k: v for k, v in p.items() if not k.startswith("ve")}, tok, tgt, 1)
    a, a0 = c["acts"][0], c0["acts"][0]
    H, hd = s.n_head, 128
    for t in range(5):
        for h in range(H):
            z = sum(a["xn1"][t, cc] * p["ve_gate"][cc, h] for cc in range(4))
            g = 3.0 / (1.0 + math.exp(-z))
            ref = a0["v"][0, h, t] + g * p["ve0"][tok[0, t], h * hd:(h + 1) * hd]
            assert np.allclose(a["v"][0, h, t], ref, rtol=1e-12, atol=1e-14), (t, h)


def test_finite_difference_with_value_embeddings():
    s, p, tok, tgt = _ve_case(depth=2, C=8, seed=5, d=256, vocab=32, seq=8)
    names = ["ve0", "ve_gate", "h0.c_qkv", "h1.c_qkv", "wte"]
    _fd_check(p, tok, tgt, s.depth, names, n_coords=6)


# --- grouped kv heads in the model -------------------------------------------

def test_gqa_model_equals_mha_with_repeated_kv_columns():
    # a q|k|v projection with Hkv kv heads gives the same loss as the full one
    # whose k and v columns repeat each kv head for its group of query heads
    s = syn.make_shape(depth=2, d_model=512, vocab=40, batch=2, seq_len=9, n_kv_head=2)
    p = syn.init_params(s, seed=3, std=0.05)
    p = {k: v.astype(np.float64) for k, v in p.items()}
    tok, tgt = syn.tokens(s, seed=4), syn.targets(s, seed=5)
    d, kvd, hd = 512, 256, 128
    full = dict(p)
    for l in range(2):
        W = p[f"h{l}.c_qkv"]
        assert W.shape == (d, d + 2 * kvd)
        rep = lambda blk: np.concatenate([blk[:, (h // 2) * hd:(h // 2 + 1) * hd] for h in range(4)], axis=1)
        full[f"h{l}.c_qkv"] = np.concatenate([W[:, :d], rep(W[:, d:d + kvd]), rep(W[:, d + kvd:])], axis=1)
    l_gqa, _ = om.forward(p, tok, tgt, 2, keep=False)
    l_mha, _ = om.forward(full, tok, tgt, 2, keep=False)
    assert abs(l_gqa - l_mha) < 1e-12


def test_finite_difference_gqa_model():
    s = syn.make_shape(depth=1, d_model=512, vocab=32, batch=1, seq_len=8, n_kv_head=2)
    p = {k: v.astype(np.float64) for k, v in syn.init_params(s, seed=6, std=0.05).items()}
    tok, tgt = syn.tokens(s, seed=7), syn.targets(s, seed=8)
    _fd_check(p, tok, tgt, 1, ["h0.c_qkv", "h0.c_proj", "wte"], n_coords=6)


def test_finite_difference_every_scalar():
    # every residual, x0, backout and smear value (3 layers: the x0 and
    # residual scales of layers past the first see streams that differ)
    s, p, tok, tgt = _extras_case(depth=3, std=0.05, seed=14, vocab=40, seq=10)
    p["scalars"] = syn.random_scalars(s, seed=15).astype(np.float64)
    _, g, _ = om.fwd_bwd(p, tok, tgt, s.depth)
    h = 1e-6
    G = g["scalars"][0]
    for j in range(p["scalars"].shape[1]):
        pp = dict(p)
        sp = p["scalars"].copy(); sp[0, j] += h; pp["scalars"] = sp
        lp, _ = om.forward(pp, tok, tgt, s.depth, keep=False)
        sm = p["scalars"].copy(); sm[0, j] -= h; pp["scalars"] = sm
        lm, _ = om.forward(pp, tok, tgt, s.depth, keep=False)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - G[j]) <= 1e-6 * max(1.0, np.abs(G).max()), (j, fd, G[j])
