"""fp64 forward and backward of the GPT decoder step (plain numpy).

TEST INFRASTRUCTURE ONLY: see the package header.

Model ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "1. Modelo GPT";
"Como Treinar Seu Próprio ChatGPT por 50 Dólares?", section "1. O Modelo
GPT"): untied token embedding and lm_head, rotary embeddings, QK
normalisation, causal attention, an MLP with ReLU^2, and (implied by the
pre-norm design and the lack of any norm gains in the optimizer table of
section "2. Optimizador Muon") gain-free RMSNorm before attention, before the
MLP and before the lm_head.  Loss: mean next-token cross-entropy over all
B*T positions.

Readings where the pages are silent (shared with the CUDA path):
  * RMSNorm eps = 1e-6, no gain.
  * RoPE: base 10000, rotate-half pairs (i, i + hd/2), angle t * base^(-2i/hd),
    out_lo = x_lo cos - x_hi sin, out_hi = x_lo sin + x_hi cos, t = position
    within the row.
  * QK norm: per-head gain-free RMSNorm applied after RoPE (the order does
    not matter mathematically: a rotation keeps the RMS).
  * attention scale 1/sqrt(hd); grouped kv heads when the fused projection
    is narrower than 3d: its columns are q (d) | k | v (Hkv * hd each), and
    query head h reads kv head h // (H / Hkv).
  * residual extras ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section
    "1. Modelo GPT", efficiency tricks 1, 2 and 3), present when params holds
    a "scalars" vector [2L + 26] = (resid lambdas [L], x0 lambdas [L],
    backout lambda, smear lambda, smear gate weights [24]):
      smear: the embedding e of position t takes gate[t] = smear_lambda *
      sigmoid(w . e[t, :24]) times the previous position's embedding,
      x[t] = e[t] + gate[t] e[t-1] (t > 0 within the sequence);
      before block i, x <- resid[i] x + x0l[i] x0 with x0 the smeared
      embedding; after the last block, x <- x - backout * x_mid with x_mid
      the residual stream entering block L // 2 (before its scaling).
    Initial values resid 1 and everything else 0 make the network the plain
    one.
  * value embeddings (section "1. Modelo GPT", value residual), present when
    params holds "ve{l}" tables [V, Hkv hd] for the layers l with l % 2 == 0
    and "ve_gate" [C, Hkv] (one block of C rows per such layer, stacked
    [n_ve * C, Hkv]): v[t, h] += 3 sigmoid(xn1[t, :C] . ve_gate_l[:, h])
    ve_l[tok[t], h*hd:(h+1)*hd] for every kv head h, xn1 being the block's
    attention input.
  * attention window per layer: full causal by default; with a layer pattern
    such as "SSSL" (section "1. Modelo GPT", sliding-window attention) the
    pattern is repeated over the layers, S = a sliding window of
    `short_window` earlier tokens, L = full causal.
  * weights are [in, out]; the fused projection's columns are q | k | v and
    head h owns columns h*hd .. h*hd+hd-1 of each.

Every intermediate is fp64; weights enter as their bf16 values.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6
ROPE_BASE = 10000.0
SMEAR_CHANNELS = 24   # embedding channels the smear gate reads


# --- building blocks -------------------------------------------------------

def rms_norm(x):
    """y = x / sqrt(mean(x^2) + eps) along the last axis; returns (y, rstd)."""
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + EPS)
    return x * rstd, rstd


def rms_norm_bwd(dy, y, rstd):
    """Gradient of the gain-free RMSNorm given its output y = x * rstd."""
    return rstd * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


def rope_angles(seq_len, head_dim):
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = ROPE_BASE ** (-2.0 * i / head_dim)
    t = np.arange(seq_len, dtype=np.float64)
    ang = np.outer(t, inv_freq)                     # [T, hd/2]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate pairs (i, i + hd/2) of x [..., T, hd] by the position angle."""
    h = x.shape[-1] // 2
    lo, hi = x[..., :h], x[..., h:]
    return np.concatenate([lo * cos - hi * sin, lo * sin + hi * cos], axis=-1)


def rope_bwd(dy, cos, sin):
    """Transpose of the rotation (rotate by the negative angle)."""
    h = dy.shape[-1] // 2
    lo, hi = dy[..., :h], dy[..., h:]
    return np.concatenate([lo * cos + hi * sin, -lo * sin + hi * cos], axis=-1)


def causal_attention(q, k, v):
    """softmax(q k^T / sqrt(hd) + causal mask) v for [B, H, T, hd]; returns (y, P)."""
    hd = q.shape[-1]
    T = q.shape[-2]
    s = np.matmul(q, np.swapaxes(k, -1, -2)) / np.sqrt(hd)
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)
    s = np.where(mask, -np.inf, s)
    s = s - np.max(s, axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return np.matmul(p, v), p


def causal_attention_bwd(dy, q, k, v, p):
    hd = q.shape[-1]
    dv = np.matmul(np.swapaxes(p, -1, -2), dy)
    dp = np.matmul(dy, np.swapaxes(v, -1, -2))
    ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True)) / np.sqrt(hd)
    dq = np.matmul(ds, k)
    dk = np.matmul(np.swapaxes(ds, -1, -2), q)
    return dq, dk, dv


def attention_hidden(T, window=None):
    """[T, T] boolean mask, True where key j is hidden from query t: j > t
    (causal) or, with a sliding window of `window` earlier tokens, j < t - window
    (so query t sees keys t - window .. t)."""
    t = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    hidden = j > t
    if window is not None:
        hidden = hidden | (j < t - window)
    return hidden


def kv_for_queries(a, n_head):
    """[B, Hkv, T, hd] -> [B, n_head, T, hd]: query head h reads kv head
    h // (n_head / Hkv) (grouped-query attention; Hkv = n_head is plain
    multi-head attention)."""
    hkv = a.shape[1]
    if n_head % hkv:
        raise ValueError(f"{n_head} query heads do not split into {hkv} kv groups")
    return np.repeat(a, n_head // hkv, axis=1)


def attention(q, k, v, window=None):
    """Causal attention with optional sliding window and grouped kv heads
    ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section "1. Modelo GPT":
    GQA and sliding-window attention, e.g. the "SSSL" layer pattern).
    q [B, H, T, hd]; k, v [B, Hkv, T, hd]; returns (y [B, H, T, hd], P)."""
    hd, T, H = q.shape[-1], q.shape[-2], q.shape[1]
    kq, vq = kv_for_queries(k, H), kv_for_queries(v, H)
    s = np.matmul(q, np.swapaxes(kq, -1, -2)) / np.sqrt(hd)
    s = np.where(attention_hidden(T, window), -np.inf, s)
    s = s - np.max(s, axis=-1, keepdims=True)
    p = np.exp(s)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return np.matmul(p, vq), p


def attention_bwd(dy, q, k, v, p):
    """(dq, dk, dv) of attention(); dk and dv add up the query heads that
    share each kv head."""
    B, H, T, hd = q.shape
    hkv = k.shape[1]
    dq, dkq, dvq = causal_attention_bwd(dy, q, kv_for_queries(k, H), kv_for_queries(v, H), p)
    g = H // hkv
    return dq, dkq.reshape(B, hkv, g, T, hd).sum(axis=2), dvq.reshape(B, hkv, g, T, hd).sum(axis=2)


def logsumexp(z):
    m = np.max(z, axis=-1, keepdims=True)
    return (m + np.log(np.sum(np.exp(z - m), axis=-1, keepdims=True)))[..., 0]


# --- the step --------------------------------------------------------------

def _split_heads(a, B, T, H, hd):
    return a.reshape(B, T, H, hd).transpose(0, 2, 1, 3)


def _merge_heads(a):
    B, H, T, hd = a.shape
    return a.transpose(0, 2, 1, 3).reshape(B * T, H * hd)


def ve_layer_count(n_layer):
    """Layers with a value embedding: l % 2 == 0."""
    return (n_layer + 1) // 2


def layer_windows(pattern, short_window, n_layer):
    """Window of every layer: pattern[l % len(pattern)] is "S" (sliding window
    of short_window earlier tokens) or "L" (full causal, None); an empty
    pattern leaves every layer full causal."""
    if not pattern:
        return [None] * n_layer
    if set(pattern) - {"S", "L"}:
        raise ValueError(f"window pattern {pattern!r} may hold only S and L")
    return [short_window if pattern[l % len(pattern)] == "S" else None for l in range(n_layer)]


def forward(params, tok, tgt, n_layer, head_dim=128, keep=True, windows=None):
    """Loss (and the saved activations) of one batch.

    params: dict of fp64-castable [in, out] matrices (wte is [V, d]).
    tok, tgt: int arrays [B, T].
    windows: per-layer attention window (None = full causal), see layer_windows.
    """
    B, T = tok.shape
    wte = np.asarray(params["wte"], dtype=np.float64)
    d = wte.shape[1]
    H = d // head_dim
    cos, sin = rope_angles(T, head_dim)
    x = wte[tok.reshape(-1)]                         # [M, d] exact row copy
    sc = params.get("scalars")
    e = x
    if sc is not None:
        sc = np.asarray(sc, dtype=np.float64).reshape(-1)
        if sc.size != 2 * n_layer + 26:
            raise ValueError("scalars must hold 2 * n_layer + 26 values")
        lam_s, w_s = sc[2 * n_layer + 1], sc[2 * n_layer + 2:]
        e3 = e.reshape(B, T, -1)
        zg = e3[:, :, :SMEAR_CHANNELS] @ w_s                 # [B, T]
        sig = 1.0 / (1.0 + np.exp(-zg))
        gate = lam_s * sig
        prev = np.concatenate([np.zeros_like(e3[:, :1]), e3[:, :-1]], axis=1)
        gate = gate * (np.arange(T) > 0)[None, :]
        x = (e3 + gate[:, :, None] * prev).reshape(B * T, -1)
    x0 = x
    x_in, x_mid = [], None
    acts = []
    for l in range(n_layer):
        if sc is not None:
            x_in.append(x)
            if l == n_layer // 2:
                x_mid = x
            x = sc[l] * x + sc[n_layer + l] * x0
        W = {n: np.asarray(params[f"h{l}.{n}"], dtype=np.float64)
             for n in ("c_qkv", "c_proj", "c_fc", "mlp_proj")}
        a = {}
        xn1, r1 = rms_norm(x)
        qkv = xn1 @ W["c_qkv"]
        # q | k | v columns; k and v have Hkv = (cols - d) / (2 hd) heads
        kvd = (qkv.shape[1] - d) // 2
        Hkv = kvd // head_dim
        q = _split_heads(qkv[:, :d], B, T, H, head_dim)
        k = _split_heads(qkv[:, d:d + kvd], B, T, Hkv, head_dim)
        v = _split_heads(qkv[:, d + kvd:], B, T, Hkv, head_dim)
        if f"ve{l}" in params:
            # value residual: v + 3 sigmoid(gate) * ve, per head
            C = params["ve_gate"].shape[0] // ve_layer_count(n_layer)
            Wg = np.asarray(params["ve_gate"], dtype=np.float64)[(l // 2) * C:(l // 2 + 1) * C]
            ve = np.asarray(params[f"ve{l}"], dtype=np.float64)[tok.reshape(-1)]      # [M, d]
            sg = 1.0 / (1.0 + np.exp(-(xn1[:, :C] @ Wg)))                           # [M, H]
            v = v + _split_heads(np.repeat(3.0 * sg, head_dim, axis=1) * ve, B, T, Hkv, head_dim)
            if keep:
                a.update(ve=ve, ve_sig=sg, ve_C=C)
        qn, rq = rms_norm(rope(q, cos, sin))
        kn, rk = rms_norm(rope(k, cos, sin))
        y, P = attention(qn, kn, v, None if windows is None else windows[l])
        ym = _merge_heads(y)
        x = x + ym @ W["c_proj"]
        xn2, r2 = rms_norm(x)
        u = xn2 @ W["c_fc"]
        h = np.maximum(u, 0.0) ** 2
        x = x + h @ W["mlp_proj"]
        if keep:
            a.update(xn1=xn1, r1=r1, qn=qn, rq=rq, kn=kn, rk=rk, v=v, P=P, ym=ym,
                     xn2=xn2, r2=r2, u=u, h=h)
        acts.append(a)
    if sc is not None:
        x = x - sc[2 * n_layer] * x_mid
    xf, rf = rms_norm(x)
    z = xf @ np.asarray(params["lm_head"], dtype=np.float64)
    lse = logsumexp(z)
    t = tgt.reshape(-1)
    row_loss = lse - z[np.arange(z.shape[0]), t]
    loss = float(np.mean(row_loss))
    cache = dict(acts=acts, xf=xf, rf=rf, z=z, lse=lse, row_loss=row_loss,
                 B=B, T=T, H=H, d=d, cos=cos, sin=sin, scalars=sc, x0=x0, x_in=x_in, x_mid=x_mid,
                 emb=e, smear_sig=sig if sc is not None else None) if keep else None
    return loss, cache


def backward(params, tok, tgt, cache, n_layer, head_dim=128):
    """Exact gradients of the mean loss w.r.t. every parameter ([in, out] layout)."""
    B, T, H, d = cache["B"], cache["T"], cache["H"], cache["d"]
    cos, sin = cache["cos"], cache["sin"]
    M = B * T
    z, lse = cache["z"], cache["lse"]
    t = tgt.reshape(-1)
    dz = np.exp(z - lse[:, None])
    dz[np.arange(M), t] -= 1.0
    dz /= M
    grads = {}
    Wlm = np.asarray(params["lm_head"], dtype=np.float64)
    grads["lm_head"] = cache["xf"].T @ dz
    dx = rms_norm_bwd(dz @ Wlm.T, cache["xf"], cache["rf"])
    sc = cache["scalars"]
    if sc is not None:
        dsc = np.zeros(2 * n_layer + 26)
        dx_final = dx                                # gradient at the backout output
        dsc[2 * n_layer] = -np.sum(cache["x_mid"] * dx_final)
        dx0 = np.zeros_like(dx)
    for l in reversed(range(n_layer)):
        a = cache["acts"][l]
        W = {n: np.asarray(params[f"h{l}.{n}"], dtype=np.float64)
             for n in ("c_qkv", "c_proj", "c_fc", "mlp_proj")}
        # MLP: x_out = x_mid + relu(rms(x_mid) Wfc)^2 Wd
        grads[f"h{l}.mlp_proj"] = a["h"].T @ dx
        dh = dx @ W["mlp_proj"].T
        du = dh * 2.0 * np.maximum(a["u"], 0.0)
        grads[f"h{l}.c_fc"] = a["xn2"].T @ du
        dx = dx + rms_norm_bwd(du @ W["c_fc"].T, a["xn2"], a["r2"])
        # attention: x_mid = x_in + attn(rms(x_in)) Wo
        grads[f"h{l}.c_proj"] = a["ym"].T @ dx
        dy = _split_heads(dx @ W["c_proj"].T, B, T, H, head_dim)
        dqn, dkn, dv = attention_bwd(dy, a["qn"], a["kn"], a["v"], a["P"])
        dq = rope_bwd(rms_norm_bwd(dqn, a["qn"], a["rq"]), cos, sin)
        dk = rope_bwd(rms_norm_bwd(dkn, a["kn"], a["rk"]), cos, sin)
        dqkv = np.concatenate([_merge_heads(dq), _merge_heads(dk), _merge_heads(dv)], axis=1)
        grads[f"h{l}.c_qkv"] = a["xn1"].T @ dqkv
        dxn1 = dqkv @ W["c_qkv"].T
        if "ve" in a:
            C, sg, ve = a["ve_C"], a["ve_sig"], a["ve"]
            dvm = _merge_heads(dv)                                                   # [M, d]
            dve = np.repeat(3.0 * sg, head_dim, axis=1) * dvm
            gve = np.zeros_like(np.asarray(params[f"ve{l}"], dtype=np.float64))
            np.add.at(gve, tok.reshape(-1), dve)
            grads[f"ve{l}"] = gve
            dgate = (ve * dvm).reshape(-1, dvm.shape[1] // head_dim, head_dim).sum(axis=-1)   # [M, Hkv]
            dz = dgate * 3.0 * sg * (1.0 - sg)
            Wg = np.asarray(params["ve_gate"], dtype=np.float64)[(l // 2) * C:(l // 2 + 1) * C]
            if "ve_gate" not in grads:
                grads["ve_gate"] = np.zeros_like(np.asarray(params["ve_gate"], dtype=np.float64))
            grads["ve_gate"][(l // 2) * C:(l // 2 + 1) * C] = a["xn1"][:, :C].T @ dz
            dxn1[:, :C] += dz @ Wg.T
        dx = dx + rms_norm_bwd(dxn1, a["xn1"], a["r1"])
        if sc is not None:
            # x' = resid[l] x_in + x0l[l] x0 (and x_in of block L // 2 feeds the backout)
            dsc[l] = np.sum(cache["x_in"][l] * dx)
            dsc[n_layer + l] = np.sum(cache["x0"] * dx)
            dx0 = dx0 + sc[n_layer + l] * dx
            dx = sc[l] * dx
            if l == n_layer // 2:
                dx = dx - sc[2 * n_layer] * dx_final
    if sc is not None:
        dx = dx + dx0
        # smear: x[t] = e[t] + lam sig(w . e[t, :24]) e[t-1]
        lam_s, w_s = sc[2 * n_layer + 1], sc[2 * n_layer + 2:]
        e3 = cache["emb"].reshape(B, T, -1)
        g3 = dx.reshape(B, T, -1)
        sig = cache["smear_sig"]
        live = (np.arange(T) > 0)[None, :]
        prev = np.concatenate([np.zeros_like(e3[:, :1]), e3[:, :-1]], axis=1)
        sdot = np.sum(g3 * prev, axis=-1) * live               # dL/dgate[t]
        de = g3.copy()
        gate = lam_s * sig * live
        de[:, :-1] += gate[:, 1:, None] * g3[:, 1:]            # e[t] is the previous token of t + 1
        dz = sdot * lam_s * sig * (1.0 - sig)
        de[:, :, :SMEAR_CHANNELS] += dz[:, :, None] * w_s[None, None, :]
        dsc[2 * n_layer + 1] = np.sum(sdot * sig)
        dsc[2 * n_layer + 2:] = np.einsum("bt,btc->c", dz, e3[:, :, :SMEAR_CHANNELS])
        dx = de.reshape(B * T, -1)
        grads["scalars"] = dsc.reshape(1, -1)
    grads["wte"] = embedding_bwd(tok, dx, params["wte"].shape[0])
    return grads


def embedding_bwd(tok, dx, vocab):
    """Gradient of the row copy x0[m] = wte[tok[m]]: row v of the result is
    the sum of dx[m] over the positions m that hold token v (zero for tokens
    that do not occur)."""
    dx = np.asarray(dx, dtype=np.float64).reshape(np.size(tok), -1)
    dwte = np.zeros((vocab, dx.shape[1]))
    np.add.at(dwte, np.asarray(tok).reshape(-1), dx)
    return dwte


def fwd_bwd(params, tok, tgt, n_layer, head_dim=128, windows=None):
    loss, cache = forward(params, tok, tgt, n_layer, head_dim, windows=windows)
    return loss, backward(params, tok, tgt, cache, n_layer, head_dim), cache
