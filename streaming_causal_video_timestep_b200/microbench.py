"""Kernel microbenchmarks through the op-level C entry points (CUDA events).

    python -m streaming_causal_video_timestep_b200.microbench attn  [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench gemm  [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench euler [--iters N]

attn : one block's attention in steady state at the 14B-like shape: 4680
       queries x 40 heads x 128 over [sink 1560 | 2 window blocks | block]
       = 15,600 keys (the per-slot launch of the stream), q pre-scaled.
gemm : the QKV projection of one block, [4680, 5120] x [15360, 5120]^T.
euler: x += dt * v over 2^20 rows x 64 fp32 (256 MB per tensor), 4 groups.
Inputs exceed L2 (126 MB) except the per-slot attention keys (160 MB K/V +
48 MB q).  Prints one JSON line per mode.
"""
from __future__ import annotations

import argparse
import json

import torch

from .stream import op_attention, op_euler, op_gemm


def _time(fn, iters, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(iters):
        fn()
    ev[1].record()
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / iters


def bench_attn(iters):
    H, d, T, F, nw = 40, 128, 4680, 1560, 2
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    rnd = lambda *s: torch.randn(*s, generator=g, device="cuda").to(torch.bfloat16)
    q = (rnd(H, T, d).float() * (1.4426950408889634 / d ** 0.5)).to(torch.bfloat16)
    ks = [rnd(H, F, d)] + [rnd(H, T, d) for _ in range(nw + 1)]
    vs = [rnd(H, F, d)] + [rnd(H, T, d) for _ in range(nw + 1)]
    out = torch.empty((T, H * d), dtype=torch.bfloat16, device="cuda")
    ms = _time(lambda: op_attention(q, ks, vs, out, q_scaled=True), iters)
    flops = 4.0 * T * (F + (nw + 1) * T) * d * H
    return {"mode": "attn", "shape": f"{T} q x {F + (nw + 1) * T} keys x {H}x{d}", "ms": round(ms, 4),
            "tflops": round(flops / ms / 1e9, 1), "flops": flops}


def bench_gemm(iters):
    M, N, K = 4680, 15360, 5120
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ms = _time(lambda: op_gemm(A, W, "store", out=out), iters)
    flops = 2.0 * M * N * K
    return {"mode": "gemm", "shape": f"{M}x{N}x{K}", "ms": round(ms, 4), "tflops": round(flops / ms / 1e9, 1),
            "flops": flops}


def bench_euler(iters):
    rows, C, G = 1 << 20, 64, 4
    x = torch.randn(rows, C, device="cuda")
    v = torch.randn(rows, C, device="cuda")
    dt = [-0.25] * G
    ms = _time(lambda: op_euler(x, v, dt, rows // G), iters)
    nbytes = 3 * rows * C * 4
    return {"mode": "euler", "shape": f"{rows}x{C} fp32", "ms": round(ms, 4), "gbs": round(nbytes / ms / 1e6, 1),
            "bytes": nbytes}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("mode", choices=["attn", "gemm", "euler", "all"])
    ap.add_argument("--iters", type=int, default=10)
    args = ap.parse_args()
    modes = ["attn", "gemm", "euler"] if args.mode == "all" else [args.mode]
    for m in modes:
        r = {"attn": bench_attn, "gemm": bench_gemm, "euler": bench_euler}[m](args.iters)
        print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
