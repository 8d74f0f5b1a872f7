"""Time single library ops on the GPU (CUDA events), e.g. for profiler captures.

    python -m gpt_pretraining_step_b200.opbench gemm --M 32768 --N 1280 --K 5120 --b-trans
    python -m gpt_pretraining_step_b200.opbench attention --B 4 --H 10 --T 2048
    python -m gpt_pretraining_step_b200.opbench newton-schulz --batch 20 --rows 1280 --cols 5120

Inputs are seeded standard normals on the device; every op runs through the
library's C ABI.  Prints one line per op with the mean time per call and the
achieved TFLOP/s of its algorithmic FLOPs.
"""
from __future__ import annotations

import argparse
import json


def _time(fn, reps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def main(argv=None):
    import torch

    from . import attention_bwd, attention_fwd, matmul_bf16, newton_schulz

    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="op", required=True)
    g = sub.add_parser("gemm", help="C[M,N] = A B (bf16 operands, fp32 out)")
    g.add_argument("--M", type=int, default=32768)
    g.add_argument("--N", type=int, default=1280)
    g.add_argument("--K", type=int, default=5120)
    g.add_argument("--a-trans", action="store_true", help="A stored [K, M]")
    g.add_argument("--b-trans", action="store_true", help="B stored [N, K]")
    a = sub.add_parser("attention", help="causal attention forward and backward, head_dim 128")
    a.add_argument("--B", type=int, default=4)
    a.add_argument("--H", type=int, default=10)
    a.add_argument("--T", type=int, default=2048)
    a.add_argument("--kv-heads", type=int, default=0, help="grouped kv heads (0 = H)")
    a.add_argument("--window", type=int, default=-1, help="sliding window, tokens of left context (-1 = full)")
    n = sub.add_parser("newton-schulz", help="five Polar Express steps on a batch of matrices")
    n.add_argument("--batch", type=int, default=20)
    n.add_argument("--rows", type=int, default=1280)
    n.add_argument("--cols", type=int, default=5120)
    n.add_argument("--tf32-steps", type=int, default=-1)
    for p in (g, a, n):
        p.add_argument("--reps", type=int, default=4)
        p.add_argument("--warmup", type=int, default=2)
    args = ap.parse_args(argv)
    torch.manual_seed(0)
    dev = "cuda"
    if args.op == "gemm":
        A = torch.randn((args.K, args.M) if args.a_trans else (args.M, args.K), device=dev).bfloat16()
        B = torch.randn((args.N, args.K) if args.b_trans else (args.K, args.N), device=dev).bfloat16()
        C = torch.empty((1, args.M, args.N), device=dev)
        ms = _time(lambda: matmul_bf16(A, B, args.M, args.N, args.K, a_trans=args.a_trans, b_trans=args.b_trans,
                                       out=C), args.reps, args.warmup)
        flops = 2.0 * args.M * args.N * args.K
        print(json.dumps({"op": "gemm", "M": args.M, "N": args.N, "K": args.K, "ms": ms,
                          "tflops": flops / (ms / 1e3) / 1e12}))
    elif args.op == "attention":
        hkv = args.kv_heads or args.H
        q = torch.randn((args.B, args.H, args.T, 128), device=dev).bfloat16()
        k, v = (torch.randn((args.B, hkv, args.T, 128), device=dev).bfloat16() for _ in range(2))
        do = torch.randn((args.B, args.T, args.H, 128), device=dev).bfloat16()
        w = args.window
        o, lse = attention_fwd(q, k, v, window=w)
        # visible (query, key) pairs: t + 1 keys for query t, at most w + 1 with a window
        pairs = sum(min(t, w) + 1 if w >= 0 else t + 1 for t in range(args.T))
        flops = 4.0 * args.B * args.H * 128 * pairs
        ms_f = _time(lambda: attention_fwd(q, k, v, window=w), args.reps, args.warmup)
        ms_b = _time(lambda: attention_bwd(q, k, v, o, lse, do, window=w), args.reps, args.warmup)
        common = {"B": args.B, "H": args.H, "kv_heads": hkv, "T": args.T, "window": w}
        print(json.dumps({"op": "attention_fwd", **common, "ms": ms_f, "tflops": flops / (ms_f / 1e3) / 1e12}))
        print(json.dumps({"op": "attention_bwd", **common, "ms": ms_b,
                          "tflops": 2.5 * flops / (ms_b / 1e3) / 1e12}))
    else:
        G = torch.randn((args.batch, args.rows, args.cols), device=dev)
        ms = _time(lambda: newton_schulz(G, tf32_steps=args.tf32_steps), args.reps, args.warmup)
        r, c = min(args.rows, args.cols), max(args.rows, args.cols)
        flops = args.batch * 5 * (r * r * c + r ** 3 + 2 * r * r * c)   # symmetric Gram and square
        print(json.dumps({"op": "newton_schulz", "batch": args.batch, "rows": args.rows, "cols": args.cols,
                          "ms": ms, "tflops": flops / (ms / 1e3) / 1e12}))


if __name__ == "__main__":
    main()
