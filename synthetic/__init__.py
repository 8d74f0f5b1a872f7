"""Seeded synthetic inputs for one GPT pretraining step.

This module is the only code that both the fp64 oracle (``oracle/``) and the
CUDA path (``gpt_pretraining_step_b200``) may use.  It holds no arithmetic of
the method: it derives tensor shapes from the depth knob, draws seeded random
numbers, and rounds float32 values to the bfloat16 grid.

Shapes follow the depth-only configuration of "¿Cómo Entrenar Tu Propio ChatGPT
por $50?" (section "La Filosofía: Un Solo Selector para Controlar Todo"):
d_model = 64 * depth, heads of dimension 128, MLP hidden 4 * d_model, vocab
32,768 (section "Lo que nanochat cubre", tokenizer row).  Weights are drawn
from N(0, 0.02) with a PCG64 generator (seed 0), tokens uniformly from
[0, vocab) (seed 1) and targets uniformly (seed 2); a Zipf(1.1) token stream
(seed 3) stands in for natural text where a skewed histogram matters.
"""
from __future__ import annotations

import dataclasses
import numpy as np

HEAD_DIM = 128
MLP_MULT = 4
VOCAB = 32768


@dataclasses.dataclass(frozen=True)
class Shape:
    depth: int
    d_model: int
    n_head: int
    head_dim: int
    mlp_hidden: int
    vocab: int
    batch: int
    seq_len: int
    n_kv_head: int = 0   # 0: as many kv heads as query heads

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len

    @property
    def kv_heads(self) -> int:
        return self.n_kv_head or self.n_head

    @property
    def qkv_cols(self) -> int:
        """Width of the fused projection: q (d) | k | v (kv_heads * head_dim each)."""
        return self.d_model + 2 * self.kv_heads * self.head_dim


def make_shape(depth: int, batch: int, seq_len: int, vocab: int = VOCAB,
               d_model: int = 0, head_dim: int = HEAD_DIM,
               mlp_mult: int = MLP_MULT, n_kv_head: int = 0) -> Shape:
    """Derive every width from ``depth`` (``d_model`` may override 64*depth)."""
    d = d_model if d_model else 64 * depth
    if d % head_dim:
        raise ValueError(f"d_model {d} is not a multiple of head_dim {head_dim}")
    if n_kv_head and (d // head_dim) % n_kv_head:
        raise ValueError(f"{n_kv_head} kv heads do not divide {d // head_dim} query heads")
    return Shape(depth=depth, d_model=d, n_head=d // head_dim, head_dim=head_dim,
                 mlp_hidden=mlp_mult * d, vocab=vocab, batch=batch, seq_len=seq_len, n_kv_head=n_kv_head)


# The workloads, named by what they are.
CONFIGS = {
    "tiny": dict(depth=2, d_model=128, vocab=512, batch=2, seq_len=64),
    "d12": dict(depth=12, batch=8, seq_len=2048),
    "d20": dict(depth=20, batch=16, seq_len=2048),
    "d24": dict(depth=24, batch=8, seq_len=2048),
    "d26": dict(depth=26, batch=8, seq_len=2048),
}


def config_shape(name: str) -> Shape:
    return make_shape(**CONFIGS[name])


def ve_layers(depth: int):
    """Layers with a value embedding (every other layer, from the first)."""
    return [l for l in range(depth) if l % 2 == 0]


def param_specs(s: Shape, extras: bool = False, ve_channels: int = 0):
    """(name, rows, cols, group) for every parameter; matrices are [in, out].

    Order: token embedding, lm_head, then per layer the fused q|k|v projection,
    the attention output projection, the MLP up projection and the MLP down
    projection.  ``group`` is the optimizer the pages route the tensor to.
    """
    d, f = s.d_model, s.mlp_hidden
    out = [("wte", s.vocab, d, "adamw"), ("lm_head", d, s.vocab, "adamw")]
    for layer in range(s.depth):
        out += [(f"h{layer}.c_qkv", d, s.qkv_cols, "muon"),
                (f"h{layer}.c_proj", d, d, "muon"),
                (f"h{layer}.c_fc", d, f, "muon"),
                (f"h{layer}.mlp_proj", f, d, "muon")]
    if extras:
        # per-layer residual and x0 scales, the backout scale, the smear scale
        # and the smear gate's 24 weights
        out.append(("scalars", 1, 2 * s.depth + 26, "adamw"))
    if ve_channels:
        # value embedding tables, then the gates of all of them stacked
        kvd = s.kv_heads * s.head_dim
        out += [(f"ve{l}", s.vocab, kvd, "adamw") for l in ve_layers(s.depth)]
        out.append(("ve_gate", ve_channels * len(ve_layers(s.depth)), s.kv_heads, "adamw"))
    return out


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-representable float32 values, as uint16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def init_params(s: Shape, seed: int = 0, std: float = 0.02, extras: bool = False, ve_channels: int = 0):
    """N(0, std) weights rounded to bf16, as float32 arrays keyed by name;
    with extras also the scalar vector at its neutral values (residual
    scales 1, everything else 0)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    params = {}
    for name, r, c, _ in param_specs(s):
        w = rng.standard_normal((r, c), dtype=np.float32) * np.float32(std)
        params[name] = round_to_bf16(w)
    if extras:
        sc = np.zeros((1, 2 * s.depth + 26), dtype=np.float32)
        sc[0, :s.depth] = 1.0
        params["scalars"] = sc
    if ve_channels:
        # value embedding tables N(0, std) like the token embedding; gates zero
        # (every gate then starts at 3 sigmoid(0) = 1.5)
        for l in ve_layers(s.depth):
            params[f"ve{l}"] = round_to_bf16(rng.standard_normal((s.vocab, s.kv_heads * s.head_dim),
                                                                 dtype=np.float32) * np.float32(std))
        params["ve_gate"] = np.zeros((ve_channels * len(ve_layers(s.depth)), s.kv_heads), dtype=np.float32)
    return params


def random_scalars(s: Shape, seed: int) -> np.ndarray:
    """Residual scales in [0.5, 1.5]; x0, backout and smear scales in
    [-0.5, 0.5]; smear gate weights N(0, 1) (the gate reads embedding
    channels of size ~0.02, so this keeps it away from saturation)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    sc = rng.uniform(-0.5, 0.5, size=(1, 2 * s.depth + 26)).astype(np.float32)
    sc[0, :s.depth] += 1.0
    sc[0, 2 * s.depth + 2:] = rng.standard_normal(24).astype(np.float32) * 10.0
    return sc


def tokens(s: Shape, seed: int = 1) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, s.vocab, size=(s.batch, s.seq_len), dtype=np.int32)


def targets(s: Shape, seed: int = 2) -> np.ndarray:
    return tokens(s, seed)


def zipf_tokens(s: Shape, seed: int = 3, a: float = 1.1) -> np.ndarray:
    """Skewed token ids: rank r drawn with probability proportional to r^-a."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ranks = np.arange(1, s.vocab + 1, dtype=np.float64)
    p = ranks ** (-a)
    p /= p.sum()
    return rng.choice(s.vocab, size=(s.batch, s.seq_len), p=p).astype(np.int32)


def gaussian(shape, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return (rng.standard_normal(shape) * std).astype(np.float32)
