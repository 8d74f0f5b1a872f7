"""The C-ABI library loads, exports every declared symbol, and its host-side
logic (configuration checks, workspace sizing, argument validation) behaves
without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gpt.h")


@pytest.fixture(scope="module")
def L():
    import gpt_pretraining_step_b200 as g
    if not os.path.exists(g.LIB_PATH):
        from gpt_pretraining_step_b200 import build
        build.build(verbose=False)
    return g.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**([a-z_][a-z0-9_]*)\s*\(", src, re.M)
    return sorted(set(n for n in names if n not in ("typedef",)))


def test_header_declares_the_step_calls():
    names = declared_functions()
    for must in ("gpt_init", "gpt_fwd_bwd", "muon_step", "adamw_step", "gpt_workspace_size"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    import gpt_pretraining_step_b200 as g
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) <= set(g.ABI_FUNCTIONS) | {"gpt_destroy"}


def _cfg(**kw):
    import gpt_pretraining_step_b200 as g
    base = dict(depth=2, batch=2, seq_len=64, vocab=512, d_model=128)
    base.update(kw)
    return g.make_config(**base)


def test_workspace_size_valid_configs(L):
    import gpt_pretraining_step_b200 as g
    p, s, a = g.workspace_size(_cfg())
    assert p > 0 and s > 0 and a > 0
    # d20: fp32 + bf16 weights of every tensor = 6 bytes/param (plus alignment)
    p20, s20, a20 = g.workspace_size(g.make_config(depth=20, batch=16, seq_len=2048))
    d, V, L_ = 1280, 32768, 20
    nparam = 2 * V * d + L_ * 12 * d * d
    assert 6 * nparam <= p20 < 6 * nparam + (1 << 20)
    # grads (4) + momentum of block matrices (4) + AdamW m, v of embeddings (8)
    assert s20 >= 4 * nparam + 4 * L_ * 12 * d * d + 8 * 2 * V * d
    assert a20 < 60 * 2 ** 30       # activations fit comfortably in 180 GB


@pytest.mark.parametrize("bad", [dict(depth=0), dict(d_model=100), dict(vocab=1001), dict(batch=0),
                                 dict(seq_len=0), dict(vocab=4), dict(window_pattern="SXL", short_window=8),
                                 dict(window_pattern="SSSL", short_window=-1),
                                 dict(window_pattern="SSSLSSSLSSSL", short_window=8), dict(ve_gate_channels=-1),
                                 dict(ve_gate_channels=129), dict(n_kv_head=3), dict(n_kv_head=-1)])
def test_workspace_size_rejects_bad_config(L, bad):
    import gpt_pretraining_step_b200 as g
    with pytest.raises(g.GptError) as e:
        g.workspace_size(_cfg(**bad))
    assert e.value.code == g.GPT_EINVAL


def test_window_pattern_configs_accepted(L):
    import gpt_pretraining_step_b200 as g
    base = g.workspace_size(_cfg())
    for pat, sw in [("SSSL", 32), ("L", 0), ("S", 0), ("", -5), ("LLS", 1 << 20)]:
        assert g.workspace_size(_cfg(window_pattern=pat, short_window=sw)) == base


def test_bad_fields_rejected(L):
    import gpt_pretraining_step_b200 as g
    for field, val in [("head_dim", 64), ("mlp_mult", 3), ("precision", 2), ("ns_tf32_steps", 6)]:
        c = _cfg()
        setattr(c, field, val)
        p = ctypes.c_size_t()
        rc = L.gpt_workspace_size(ctypes.byref(c), ctypes.byref(p), ctypes.byref(p), ctypes.byref(p))
        assert rc == g.GPT_EINVAL, field
        assert L.gpt_last_error()


def test_null_arguments_are_einval(L):
    import gpt_pretraining_step_b200 as g
    assert L.gpt_fwd_bwd(None, None, None, None, 0) == g.GPT_EINVAL
    assert L.muon_step(None, 0.02, 0.95, 0.0) == g.GPT_EINVAL
    assert L.muon_step_normuon(None, 0.02, 0.95, 0.0, 0.95) == g.GPT_EINVAL
    assert L.muon_step_layers(None, 0.02, 0.95, 0.0, -1.0, 0, 1) == g.GPT_EINVAL
    assert L.gpt_block_region(None, 0, 0, 0, 1, None, None) == g.GPT_EINVAL
    assert L.gpt_set_adam_step(None, 3) == g.GPT_EINVAL
    assert L.gpt_get_adam_step(None, None) == g.GPT_EINVAL
    assert L.adamw_step(None, 1e-3, 0.8, 0.95, 1e-10, 0.0) == g.GPT_EINVAL
    assert L.gpt_check(None) == g.GPT_EINVAL
    assert L.gpt_num_tensors(None) == 0
    out = ctypes.c_void_p()
    c = _cfg()
    assert L.gpt_init(ctypes.byref(c), None, None, None, None, ctypes.byref(out)) == g.GPT_EINVAL
    # misaligned buffers are refused before any device work
    assert L.gpt_init(ctypes.byref(c), ctypes.c_void_p(8), ctypes.c_void_p(256), ctypes.c_void_p(512), None,
                      ctypes.byref(out)) == g.GPT_EINVAL
    assert L.gpt_op_matmul_bf16(None, None, None, 1, 1, 1, 1, 0, 0, None) == g.GPT_EINVAL
    assert L.gpt_op_newton_schulz(None, None, 1, 8, 8, 0, None, None) == g.GPT_EINVAL


def test_split_plan_matches_header_contract(L):
    # the scratch query is pure host arithmetic
    assert L.gpt_op_newton_schulz_scratch(2, 128, 384) > 2 * 128 * 384 * 4 * 2


def test_workspace_sizes_follow_the_options(L):
    """Grouped kv heads shrink the q|k|v parameters; value embeddings add
    their tables; the residual extras add their saved streams."""
    import gpt_pretraining_step_b200 as g
    base = dict(depth=4, batch=2, seq_len=64, vocab=512, d_model=512)
    p0, s0, a0 = g.workspace_size(g.make_config(**base))
    p1, s1, a1 = g.workspace_size(g.make_config(**base, n_kv_head=1))
    d, L = 512, 4
    # q|k|v goes from [d, 3d] to [d, d + 256] per layer: fp32 master + bf16 copy
    assert p0 - p1 >= 6 * L * d * (3 * d - (d + 256)) - 256 * 16
    assert s1 < s0 and a1 < a0
    p2, s2, a2 = g.workspace_size(g.make_config(**base, ve_gate_channels=8))
    n_ve = (L + 1) // 2
    slack = 4096                                # small placeholder allocations when an option is off
    assert p2 - p0 >= 6 * n_ve * 512 * d - slack        # tables: fp32 master + bf16 copy
    assert s2 - s0 >= 12 * n_ve * 512 * d - slack       # gradient + AdamW m, v
    p3, s3, a3 = g.workspace_size(g.make_config(**base, residual_extras=True))
    assert a3 - a0 >= 4 * L * 2 * 64 * d        # the saved block inputs, fp32
