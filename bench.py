#!/usr/bin/env python
"""Training-step benchmark: tokens/s and MFU of one GPT pretraining step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config d20] [--impl ours|reference]

A step is the whole hot path on one batch of synthetic input: forward and
backward of the decoder, the Muon update of every block matrix and the AdamW
update of the embedding and lm_head, all through libgpt's C ABI.  Inputs are
resident in HBM when the timed region starts; the activations (tens of GB)
exceed the 126 MB L2 many times over, so no L2 flush is needed between steps.
For N > 1 (launched by torch.distributed.run) every rank trains on its own
batch and the gradients are averaged with one NCCL all-reduce per step before
the (replicated) optimizer step, or, with --shard-optimizer, exchanged in three
phases around a Muon step split by layer; the reported time is the max over
ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
on a bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "training tokens/sec and MFU (fwd+bwd+Muon step) on 1 B200, d20 seq 2048 bf16"
N_BATCHES = 4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="d20", choices=["d12", "d20", "d24", "d26"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ns-tf32-steps", type=int, default=-1,
                    help="Newton-Schulz operand precision: -1 = fp16 (default), 0..5 = leading tf32 steps, then bf16")
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: forward block projections on e4m3 operands")
    ap.add_argument("--normuon", type=float, default=None, metavar="BETA2",
                    help="NorMuon variance reduction on the Muon updates with this second-moment decay")
    ap.add_argument("--window-pattern", default="", help='per-layer attention windows, e.g. "SSSL" (S = sliding)')
    ap.add_argument("--short-window", type=int, default=1024, help="left context of an S layer, tokens")
    ap.add_argument("--residual-extras", action="store_true",
                    help="per-layer residual / x0 scales and backout (scalar parameters trained by AdamW)")
    ap.add_argument("--value-embeds", type=int, default=0, metavar="C",
                    help="value embeddings on layers 0, 2, ... with C gate channels (0 = off)")
    ap.add_argument("--shard-optimizer", action="store_true",
                    help="N > 1: each rank runs Muon on its own layer range (three-phase ZeRO-2 style exchange)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--breakdown", action="store_true", help="per-category device times in the JSON line")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)
    return a


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ FLOPs

def model_flops_per_token(s, causal=False):
    """PaLM-style model FLOPs per token: 6 N_matmul + 12 L d T (embeddings
    excluded); with causal=True the attention term counts only the half of the
    score matrix that the causal mask keeps (6 L d T)."""
    n_matmul = s.depth * 12 * s.d_model ** 2 + s.d_model * s.vocab
    return 6 * n_matmul + (6 if causal else 12) * s.depth * s.d_model * s.seq_len


def category_work(s):
    """Algorithmic FLOPs (tensor categories) or bytes (HBM categories) per step."""
    M, d, F, V, L, B, H, T = s.tokens, s.d_model, s.mlp_hidden, s.vocab, s.depth, s.batch, s.n_head, s.seq_len
    causal = B * H * 128 * T * (T + 1) / 2          # q.k products that the causal mask keeps
    r = d
    ns = 0.0
    for nmat, c in ((L, 3 * d), (L, d), (2 * L, F)):
        ns += nmat * 5 * (r * r * c + r ** 3 + 2 * r * r * c)   # symmetric Gram and square, dense update
    return {
        "qkv_gemm": ("tensor", 2 * M * d * 3 * d * L),
        "proj_gemm": ("tensor", 2 * M * d * d * L),
        "fc_gemm": ("tensor", 2 * M * d * F * L),
        "down_gemm": ("tensor", 2 * M * F * d * L),
        "attn_fwd": ("tensor", 4 * causal * L),
        "attn_bwd": ("tensor", 10 * causal * L),
        "logits_gemm": ("tensor", 2 * M * d * V),
        "lm_dx_gemm": ("tensor", 2 * M * d * V),
        "lm_dw_gemm": ("tensor", 2 * M * d * V),
        "dx_gemm": ("tensor", 24 * M * d * d * L),
        "dw_gemm": ("tensor", 24 * M * d * d * L),
        "ns_gemm": ("tensor", ns),
        # bytes: read fp32 x, write bf16 y (+ rstd) forward; read fp32 dy, bf16 y,
        # fp32 dx, write fp32 dx and bf16 dx backward
        "norm": ("hbm", (2 * L + 1) * M * d * 6 + (2 * L + 1) * M * d * 14),
        "ce_finish": ("hbm", M * V * 2 * 2),
        # q only (the attention backward writes the k and v columns): read fp32
        # dq and bf16 q, write bf16
        "qk_bwd": ("hbm", L * M * d * (4 + 2 + 2)),
        "embed": ("hbm", M * d * (2 + 4) + M * d * 4 + V * d * 4),
        "muon_elem": ("hbm", L * 12 * d * d * (12 + 4 + 4 + 10)),
        "adamw": ("hbm", 2 * V * d * 30),
    }


def fp8_fraction(category, s):
    """Share of a category's FLOPs that run on e4m3 operands with --precision fp8:
    the attention output, MLP up and MLP down projections in all three of their
    GEMMs (forward, activation gradient, weight gradient); q|k|v, attention,
    the lm_head and Newton-Schulz stay 16-bit.  Per layer and token the block
    dX (and dW) GEMMs take 2 d (d + 2 F) FLOPs on e4m3 against 2 d qkv_cols
    for q|k|v (18 of 24 d^2 with F = 4 d and full kv heads)."""
    if category in ("proj_gemm", "fc_gemm", "down_gemm"):
        return 1.0
    if category in ("dx_gemm", "dw_gemm"):
        e4m3 = s.d_model * (s.d_model + 2 * s.mlp_hidden)
        return e4m3 / (e4m3 + s.d_model * s.qkv_cols)
    return 0.0


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.file.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- CPU oracle

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def _layer_params(params, layers):
    """The embedding, lm_head and the first `layers` blocks of a parameter set."""
    keep = {"wte", "lm_head"} | {f"h{l}.{n}" for l in range(layers) for n in ("c_qkv", "c_proj", "c_fc", "mlp_proj")}
    return {k: v for k, v in params.items() if k in keep}


class OracleSampler:
    """Times the fp64 oracle on bounded samples of one step, at the step's real
    sequence length, and scales them to the whole step.

    Samples: the forward+backward of the head alone (embedding, final norm,
    lm_head, cross-entropy) on one sequence of T tokens, and of the head plus
    one decoder block on the same sequence (their difference is one block's
    time, attention's T^2 term included); Newton-Schulz + Muon on one matrix
    of a block-matrix kind; AdamW on a fraction of the embedding.  The step
    estimate is B (L t_block + t_head) + sum over kinds of (matrices of the
    kind) t_muon + t_adamw scaled to the embedding and lm_head.
    """

    KINDS = ("c_qkv", "c_proj", "c_fc", "mlp_proj")

    def __init__(self, s, seed=0, adam_frac=1 / 32):
        from oracle import model as om
        from oracle import optim as oo
        self.om, self.oo = om, oo
        self.s = s
        self.params = _layer_params(syn.init_params(syn.make_shape(depth=1, batch=1, seq_len=s.seq_len,
                                                                   vocab=s.vocab, d_model=s.d_model), seed=seed), 1)
        self.tok = syn.tokens(s)[:1]
        self.tgt = syn.targets(s)[:1]
        self.adam_frac = adam_frac
        self.times = {}

    def run(self, what):
        """Run one sample ("head", "block", "muon:<kind>" or "adamw"); returns its seconds."""
        import numpy as np
        om, oo, p = self.om, self.oo, self.params
        t0 = time.perf_counter()
        if what == "head":
            om.fwd_bwd(_layer_params(p, 0), self.tok, self.tgt, 0)
        elif what == "block":
            om.fwd_bwd(p, self.tok, self.tgt, 1)
        elif what.startswith("muon:"):
            W = p[f"h0.{what[5:]}"].astype(np.float64)
            G = syn.gaussian(W.shape, seed=5)
            oo.muon_step(W, G, np.zeros_like(W), 0.02)
        elif what == "adamw":
            n = int(self.s.vocab * self.s.d_model * self.adam_frac)
            pp = p["wte"].ravel()[:n].astype(np.float64)
            oo.adamw_step(pp, syn.gaussian((n,), seed=6).astype(np.float64), np.zeros(n), np.zeros(n), 1, 3e-3)
        else:
            raise ValueError(what)
        dt = time.perf_counter() - t0
        self.times.setdefault(what, []).append(dt)
        return dt

    def schedule(self):
        return ["head", "block"] + [f"muon:{k}" for k in self.KINDS] + ["adamw"]

    def step_seconds(self):
        s, t = self.s, {k: statistics.mean(v) for k, v in self.times.items()}
        block = max(t["block"] - t["head"], 0.0)
        nmat = {"c_qkv": s.depth, "c_proj": s.depth, "c_fc": s.depth, "mlp_proj": s.depth}
        muon = sum(nmat[k] * t[f"muon:{k}"] for k in self.KINDS)
        return s.batch * (s.depth * block + t["head"]) + muon + t["adamw"] * 2 / self.adam_frac

    def describe(self):
        s = self.s
        return (f"fp64 oracle at T={s.seq_len}: fwd+bwd of the head alone and of the head plus one block on one "
                f"sequence (block time = difference, scaled x{s.depth} blocks x{s.batch} sequences), Muon on one "
                f"matrix per kind (x{s.depth} each), AdamW on {self.adam_frac:.4f} of the embedding (scaled to wte "
                f"and lm_head)")


def oracle_sample(s):
    """(step seconds, description, threads, seconds of CPU work) for the cpu_baseline."""
    o = OracleSampler(s)
    spent = sum(o.run(w) for w in o.schedule())
    return o.step_seconds(), o.describe(), _oracle_threads(), spent


def bench_config(a, s, world):
    """The `config` object of both arms' JSON lines (the same workload)."""
    return {"workload": f"{a.config} GPT step (fwd+bwd+{optim_name(a)}+AdamW)", "global_batch": s.batch * world,
            "seq_len": s.seq_len, "depth": s.depth, "d_model": s.d_model, "vocab": s.vocab,
            "precision": a.precision,
            "parallelism": f"dp{world}" + ("+sharded-optimizer" if a.shard_optimizer and world > 1 else ""),
            "ns_operands": "fp16" if a.ns_tf32_steps < 0 else f"tf32 x{a.ns_tf32_steps} + bf16",
            "l2": "no flush: step working set (activations ~20 GB) far exceeds the 126 MB L2",
            "attention": (f"windows {a.window_pattern} (S = {a.short_window} tokens)" if a.window_pattern
                          else "full causal"),
            "residual_extras": bool(a.residual_extras), "value_embed_channels": a.value_embeds,
            "batches": f"{N_BATCHES} resident seeded batches, used in turn"}


def run_reference(a):
    """The oracle as the reference arm: each step is one bounded sample of the
    workload (the samples of OracleSampler in turn), timed for real; `value`
    is the workload's tokens/s estimated from the mean time of each sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = syn.config_shape(a.config)
    o = OracleSampler(s, adam_frac=1 / 256)
    sched = o.schedule()
    # each step runs every sample once; warm-up steps are discarded
    for _ in range(a.warmup):
        for w in sched:
            o.run(w)
    o.times = {}
    timed = [sum(o.run(w) for w in sched) for _ in range(a.steps)]
    ms = statistics.mean(timed) * 1e3
    value = s.tokens / o.step_seconds()
    sample = o.describe() + (f"; each timed step runs every sample once ({a.steps} steps, {sum(timed):.1f} s of "
                             f"CPU work); value = tokens of the workload's step / its estimated time")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(a, s, 1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "estimated_step_seconds": o.step_seconds(),
    }), flush=True)


# --------------------------------------------------------------- GPU arm

def run_ours(a):
    import numpy as np
    import torch
    import torch.distributed as dist

    import gpt_pretraining_step_b200 as g
    from gpt_pretraining_step_b200 import dp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    g.lib()
    s = syn.config_shape(a.config)
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    st = g.GPTStep(depth=s.depth, batch=s.batch, seq_len=s.seq_len, vocab=s.vocab, d_model=s.d_model,
                   ns_tf32_steps=a.ns_tf32_steps, seed=1234, stream=stream,
                   precision=1 if a.precision == "fp8" else 0, window_pattern=a.window_pattern,
                   short_window=a.short_window, residual_extras=a.residual_extras, ve_gate_channels=a.value_embeds)
    # a few resident seeded batches used in turn, so the printed loss is not
    # the loss of one memorised batch
    batches = [(torch.tensor(syn.tokens(s, seed=dp.rank_seed(1 + 100 * i, rank))).cuda(),
                torch.tensor(syn.targets(s, seed=dp.rank_seed(2 + 100 * i, rank))).cuda()) for i in range(N_BATCHES)]
    grads = st.grad_view() if world > 1 else None
    hp = dict(muon=(0.02, 0.95, 0.0), adam=(3e-3, 0.8, 0.95, 1e-10, 0.0))
    counter = [0]
    # the pages' ZeRO-2 exchange: bucket reduces overlapped with the backward,
    # Muon by layer ranges, AdamW by rows
    ex = dp.ShardedExchange(st, s.depth, s.vocab, s.d_model) if a.shard_optimizer and world > 1 else None

    def step():
        tok, tgt = batches[counter[0] % N_BATCHES]
        counter[0] += 1
        if ex is not None:
            ex.step(tok, tgt, muon=hp["muon"], adam=hp["adam"], normuon_beta2=-1.0 if a.normuon is None else a.normuon)
            return
        st.fwd_bwd(tok, tgt)
        if grads is not None:
            dp.average_gradients(grads)
        if a.normuon is None:
            st.muon_step(*hp["muon"])
        else:
            st.muon_step_normuon(*hp["muon"], a.normuon)
        st.adamw_step(*hp["adam"])

    # warm-up; the first step's loss is kept (the initial weights give a known
    # value) and the last warm-up step records every launch category
    first_loss = None
    for i in range(a.warmup):
        if i == a.warmup - 1:
            st.profile_enable(g.PROF_CATEGORIES)
        step()
        if i == 0:
            first_loss = float(st.loss[0].item())
    torch.cuda.synchronize()
    st.check()
    prof = st.profile_read()
    work = category_work(s)
    dominant = max(prof, key=lambda c: prof[c][0]) if prof else None
    st.profile_enable([dominant] if dominant else [])

    pk, pk_src = peaks()
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    n0 = st.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(a.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    launches = st.launch_count() - n0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = dp.max_over_ranks(ev0.elapsed_time(ev1) / a.steps, device="cuda")
    st.check()
    live = st.profile_read()
    st.profile_enable([])
    loss = float(st.loss[0].item())

    tokens_per_step = s.tokens * world
    value = tokens_per_step / (ms / 1e3)
    fpt = model_flops_per_token(s)
    mfu_sust = fpt * s.tokens / (ms / 1e3) / (pk["bf16_tflops_sustained"] * 1e12)
    mfu_nominal = fpt * s.tokens / (ms / 1e3) / 2.25e15
    mfu_causal = model_flops_per_token(s, causal=True) * s.tokens / (ms / 1e3) / (pk["bf16_tflops_sustained"] * 1e12)

    roof = None
    if dominant and dominant in live and live[dominant][1]:
        kind, amount = work[dominant]
        per_launch_ms = live[dominant][0] / live[dominant][1]
        per_launch_work = amount / (live[dominant][1] / a.steps)
        if kind == "tensor":
            achieved = per_launch_work / (per_launch_ms / 1e3) / 1e12
            peak = pk["bf16_tflops_sustained"]
            src = f"{pk_src} bf16_tflops_sustained"
            f8 = fp8_fraction(dominant, s) if a.precision == "fp8" else 0.0
            if f8 > 0:
                # the category's fp8 FLOPs against twice the bf16 figure (the nominal
                # dense ratio), the rest against the bf16 figure
                peak = 1.0 / ((1.0 - f8) / peak + f8 / (2.0 * peak))
                src += f" blended with 2x for the fp8 share ({f8:.2f} of the FLOPs)"
            # DRAM traffic needs hardware counters (an ncu capture), which a timed
            # run does not take: reported as null here
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None, "kernel": dominant, "peak_source": src}
        else:
            achieved = per_launch_work / (per_launch_ms / 1e3) / 1e9
            peak = pk["hbm_gbs"]
            roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "traffic": None, "kernel": dominant, "peak_source": f"{pk_src} hbm_gbs"}

    breakdown = {}
    if True:
        for c, (tms, n) in sorted(prof.items(), key=lambda kv: -kv[1][0]):
            kind, amount = work.get(c, ("", 0))
            e = {"ms": round(tms, 3), "launches": n}
            if tms > 0 and amount:
                if kind == "tensor":
                    e["tflops"] = round(amount / (tms / 1e3) / 1e12, 1)
                else:
                    e["gbs"] = round(amount / (tms / 1e3) / 1e9, 1)
            breakdown[c] = e

    # device time of the optimizer calls (Newton-Schulz, Muon elementwise, AdamW)
    # against the rest of the step
    opt_ms = sum(prof.get(c, (0.0, 0))[0] for c in ("ns_gemm", "muon_elem", "adamw"))
    split = {"optimizer_ms": round(opt_ms, 3), "fwd_bwd_ms": round(ms - opt_ms, 3)} if prof else None
    if split and a.precision == "fp8":
        # against the fp8 dense peak (twice the measured bf16 figure, the nominal ratio)
        split["mfu_vs_fp8_peak"] = mfu_sust / 2

    e2e = None
    if not a.no_e2e:
        e2e = run_e2e(a, st, s, rank, world, grads, stream, ex)
        if world > 1:
            e2e["ms_per_step"] = dp.max_over_ranks(e2e["ms_per_step"], device="cuda")
            e2e["value"] = tokens_per_step / (e2e["ms_per_step"] / 1e3)

    # Newton-Schulz over every block matrix on its own (the Muon step without
    # the forward and backward), timed with events on the library's stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.profile_enable(["ns_gemm"])
    e0.record(stream)
    st.muon_step(*hp["muon"])
    e1.record(stream)
    torch.cuda.synchronize()
    ns_prof = st.profile_read()
    st.profile_enable([])
    ns_ms = ns_prof.get("ns_gemm", (0.0, 0))[0]
    ns_alone = {"muon_step_ms": e0.elapsed_time(e1), "newton_schulz_ms": ns_ms,
                "newton_schulz_tflops": work["ns_gemm"][1] / (ns_ms / 1e3) / 1e12 if ns_ms > 0 else None,
                "matrices": 4 * s.depth,
                "shapes": [[s.d_model, s.qkv_cols], [s.d_model, s.d_model], [s.d_model, s.mlp_hidden],
                           [s.mlp_hidden, s.d_model]]}
    sig2 = 0.02 ** 2 * s.d_model
    first_loss_expect = math.log(s.vocab) + sig2 / 2 - (math.exp(sig2) - 1) / (2 * s.vocab)
    clock_peak = None
    if clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        clock_peak = 2.25e15 * clocks["sm_mhz"] / clocks["sm_max_mhz"]

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        step_s, desc, threads, spent = oracle_sample(s)
        cpu = {"value": s.tokens / step_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": desc + f" ({spent:.1f} s of CPU work)"}

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if a.precision == "bf16" else "bf16+e4m3", "data": "synthetic",
            "config": bench_config(a, s, world),
            "mfu": mfu_sust, "mfu_vs_nominal_2250": mfu_nominal,
            "mfu_vs_dense_at_sampled_clock": (fpt * s.tokens / (ms / 1e3) / clock_peak) if clock_peak else None,
            "first_step_loss": first_loss, "first_step_loss_closed_form": first_loss_expect,
            "first_step_loss_ok": (first_loss is not None and
                                   abs(first_loss - first_loss_expect) / first_loss_expect <= 1e-2),
            "newton_schulz_alone": ns_alone,
            "mfu_peak": f"{pk_src} bf16_tflops_sustained {pk['bf16_tflops_sustained']}",
            "model_tflop_per_step": fpt * s.tokens / 1e12,
            "mfu_attention_causal_half": mfu_causal,
            "loss": loss, "clocks": clocks, "gpu_launches": launches, "roofline": roof, "cpu_baseline": cpu,
            "e2e": None if e2e is None else {k: e2e[k] for k in ("value", "unit", "h2d_bytes_per_step",
                                                                 "d2h_bytes_per_step")},
            "breakdown_ms_per_step_category": breakdown,
            "step_split": split,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(a, st, s, rank, world, grads, stream, ex=None):
    """Whole steps through the public API from host buffers: H2D of tokens and
    targets from pinned memory, the step, D2H of the loss, all timed.  One GPU
    uses the single host-buffer entry point; data-parallel ranks compose the
    public calls with the gradient all-reduce in between."""
    import torch
    import torch.distributed as dist

    import gpt_pretraining_step_b200 as g
    from gpt_pretraining_step_b200 import dp
    tok = torch.tensor(syn.tokens(s, seed=dp.rank_seed(11, rank))).pin_memory()
    tgt = torch.tensor(syn.targets(s, seed=dp.rank_seed(12, rank))).pin_memory()
    hp = g.HParams(muon_lr=0.02, muon_momentum=0.95, muon_wd=0.0, adam_lr=3e-3, adam_beta1=0.8, adam_beta2=0.95,
                   adam_eps=1e-10, adam_wd=0.0)
    dtok = torch.empty_like(tok, device="cuda")
    dtgt = torch.empty_like(tgt, device="cuda")
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()

    def one():
        if world == 1 and a.normuon is None:
            return st.train_step_host(tok, tgt, hp)
        dtok.copy_(tok, non_blocking=True)
        dtgt.copy_(tgt, non_blocking=True)
        if ex is not None:
            loss = ex.step(dtok, dtgt, muon=(hp.muon_lr, hp.muon_momentum, hp.muon_wd),
                           adam=(hp.adam_lr, hp.adam_beta1, hp.adam_beta2, hp.adam_eps, hp.adam_wd),
                           normuon_beta2=-1.0 if a.normuon is None else a.normuon)
            loss_host.copy_(loss.reshape(1), non_blocking=True)
            stream.synchronize()
            return float(loss_host[0])
        loss = st.fwd_bwd(dtok, dtgt)
        dp.average_gradients(grads)
        if a.normuon is None:
            st.muon_step(hp.muon_lr, hp.muon_momentum, hp.muon_wd)
        else:
            st.muon_step_normuon(hp.muon_lr, hp.muon_momentum, hp.muon_wd, a.normuon)
        st.adamw_step(hp.adam_lr, hp.adam_beta1, hp.adam_beta2, hp.adam_eps, hp.adam_wd)
        loss_host.copy_(loss.reshape(1), non_blocking=True)
        stream.synchronize()
        return float(loss_host[0])

    one()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        one()
    dt = (time.perf_counter() - t0) / a.steps
    return {"value": s.tokens / dt, "unit": "tokens/s", "ms_per_step": dt * 1e3,
            "h2d_bytes_per_step": int(tok.numel() * 4 + tgt.numel() * 4), "d2h_bytes_per_step": 4}


def optim_name(a):
    return "Muon" if a.normuon is None else f"NorMuon(beta2={a.normuon})"


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
