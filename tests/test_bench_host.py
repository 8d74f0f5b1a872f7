"""Host-side accounting of bench.py (CPU only): the model FLOPs behind the
MFU, the per-category algorithmic work behind the roofline, the clock-record
parsing behind the rejection rule, and the warm-up floor."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synthetic as syn  # noqa: E402


def test_d20_model_flops_per_step():
    # 6 N_matmul + 12 L d T per token over 16 x 2048 tokens: 106.17 TFLOP
    s = syn.config_shape("d20")
    n_matmul = 20 * 12 * 1280 ** 2 + 1280 * 32768
    assert bench.model_flops_per_token(s) == 6 * n_matmul + 12 * 20 * 1280 * 2048
    assert abs(bench.model_flops_per_token(s) * s.tokens / 1e12 - 106.17) < 0.01
    # the causal variant halves only the attention term
    assert bench.model_flops_per_token(s) - bench.model_flops_per_token(s, causal=True) == 6 * 20 * 1280 * 2048


@pytest.mark.parametrize("name", ["d12", "d20", "d24", "d26"])
def test_projection_categories_add_up_to_the_matmul_flops(name):
    # forward projections, their dX and dW GEMMs and the three lm_head GEMMs are
    # exactly 6 N_matmul per token; attention and Newton-Schulz come on top
    s = syn.config_shape(name)
    w = bench.category_work(s)
    proj = ["qkv_gemm", "proj_gemm", "fc_gemm", "down_gemm", "dx_gemm", "dw_gemm", "logits_gemm", "lm_dx_gemm",
            "lm_dw_gemm"]
    assert all(w[c][0] == "tensor" for c in proj)
    total = sum(w[c][1] for c in proj)
    n_matmul = s.depth * 12 * s.d_model ** 2 + s.d_model * s.vocab
    assert total == 6 * n_matmul * s.tokens
    # the backward of attention is counted as 2.5 forwards
    assert w["attn_bwd"][1] == 2.5 * w["attn_fwd"][1]


def test_fp8_share_of_the_block_gradient_gemms():
    # with F = 4 d and full kv heads the e4m3 projections (attention output, MLP
    # up, MLP down) are 18 of the 24 d^2 FLOPs per token of the block dX and dW
    # GEMMs; the forward projection categories are wholly fp8 or wholly 16-bit
    s = syn.config_shape("d26")
    assert abs(bench.fp8_fraction("dx_gemm", s) - 18 / 24) < 1e-12
    assert bench.fp8_fraction("dw_gemm", s) == bench.fp8_fraction("dx_gemm", s)
    assert bench.fp8_fraction("fc_gemm", s) == 1.0 and bench.fp8_fraction("qkv_gemm", s) == 0.0
    assert bench.fp8_fraction("attn_bwd", s) == 0.0 and bench.fp8_fraction("ns_gemm", s) == 0.0
    # the share matches the per-category work: proj + fc + down over all four
    w = bench.category_work(s)
    fp8_fwd = w["proj_gemm"][1] + w["fc_gemm"][1] + w["down_gemm"][1]
    assert abs(fp8_fwd / (fp8_fwd + w["qkv_gemm"][1]) - bench.fp8_fraction("dx_gemm", s)) < 1e-12


def test_clock_record_parsing_and_reasons(tmp_path):
    sampler = bench.ClockSampler(0)

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    sampler.proc = Done()
    rows = ["0, 1500, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1520, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1980, 1965, 700.0, 0x0, Not Active, Active, Not Active, Not Active",
            "garbage line"]
    sampler.file.write("\n".join(rows) + "\n")
    out = sampler.stop()
    assert out["sm_mhz"] == 1520.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_warmup_floor(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "1", "--steps", "2"])
    a = bench.parse()
    assert a.warmup == 3 and a.steps == 2 and a.gpus == 1 and a.impl == "ours"
