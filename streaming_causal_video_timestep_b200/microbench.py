"""Kernel microbenchmarks through the op-level C entry points (CUDA events).

    python -m streaming_causal_video_timestep_b200.microbench attn  [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench gemm  [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench gemm_out [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench euler [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench rerope [--iters N] [--layers L]
    python -m streaming_causal_video_timestep_b200.microbench gemm_fp8 [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench attn_fp8 [--iters N]
    python -m streaming_causal_video_timestep_b200.microbench qkv_stream [--iters N] [--fp8]

attn : one block's attention in steady state at the 14B-like shape: 4680
       queries x 40 heads x 128 over [sink 1560 | 2 window blocks | block]
       = 15,600 keys (the per-slot launch of the stream), q pre-scaled.
attn_fp8: the same attention on e4m3 q/K/V (per-head scales, e4m3 P).
gemm : the QKV projection of one block, [4680, 5120] x [15360, 5120]^T.
gemm_out: the output projection of the 4-slot grouped launch, [18720, 5120] x
       [5120, 5120]^T, with the residual epilogue and with a plain bf16 store.
euler: x += dt * v over 2^20 rows x 64 fp32 (256 MB per tensor), 4 groups.
gemm_fp8: the QKV projection shape on e4m3 operands (kind::f8f6f4, per-row
       scales, bf16 output), and the per-row quantization of its activation.
rerope: the per-block sink re-rope of the 8-sublayer stream (30x52 grid, 40x128
       heads, 4 slots), one launch a tick for all layers: reads each layer's
       fp32 un-roped sink K (32 MB) once and writes 4 bf16 roped copies (64 MB),
       766 MB a launch; timed by the stream's profiling counters.
qkv_stream: the QKV projection with its fused RoPE / ring-append epilogue and
       the output projection with its residual epilogue, as they run in the
       4-slot grouped stream ([18720, 5120] x [15360, 5120]^T and x [5120,
       5120]^T), in a one-sublayer stream at the 14B-like shape; bf16, or with
       --fp8 on e4m3 operands; timed by the stream's profiling counters.
Inputs exceed L2 (126 MB) except the per-slot attention keys (160 MB K/V +
48 MB q).  Each timed loop spans at least 1.5 s; prints one JSON line per mode
with the SM clock record (median under load, throttle reasons) taken around it.
"""
from __future__ import annotations

import argparse
import json

import torch

from .clocks import ClockSampler
from .stream import op_attention, op_attention_fp8, op_euler, op_gemm, op_gemm_fp8, op_quantize_e4m3


def _time(fn, iters, warmup=3, min_ms=1500.0):
    """Average ms of fn on the current stream (CUDA events), after warm-up; at
    least `iters` launches and enough of them to span min_ms, so that the clock
    sampler running around each mode sees several samples under load."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    fn()
    ev[1].record()
    torch.cuda.synchronize()
    n = max(iters, int(min_ms / max(ev[0].elapsed_time(ev[1]), 1e-3)) + 1)
    ev[0].record()
    for _ in range(n):
        fn()
    ev[1].record()
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / n


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


def bench_attn_fp8(iters):
    H, d, T, F, nw = 40, 128, 4680, 1560, 2
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    rnd = lambda *s: torch.randn(*s, generator=g, device="cuda").to(torch.float8_e4m3fn).view(torch.uint8)
    q = rnd(H, T, d)
    ks = [rnd(H, F, d)] + [rnd(H, T, d) for _ in range(nw + 1)]
    vs = [rnd(H, F, d)] + [rnd(H, T, d) for _ in range(nw + 1)]
    sq = torch.ones(H, device="cuda")
    sk = torch.ones(H, device="cuda")
    sv = torch.ones(H, device="cuda")
    out = torch.empty((T, H * d), dtype=torch.bfloat16, device="cuda")
    ms = _time(lambda: op_attention_fp8(q, ks, vs, sq, sk, sv, out), iters)
    flops = 4.0 * T * (F + (nw + 1) * T) * d * H
    return {"mode": "attn_fp8", "shape": f"{T} q x {F + (nw + 1) * T} keys x {H}x{d} e4m3", "ms": round(ms, 4),
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


def bench_gemm_out(iters):
    """The output projection of the grouped 4-slot stream (M = 4 x 4680), with the
    residual epilogue it runs with there (h32 += A W^T, plus the bf16 copy) and,
    for comparison, with a plain bf16 store."""
    M, N, K = 4 * 4680, 5120, 5120
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    h32 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    flops = 2.0 * M * N * K
    res = {"mode": "gemm_out", "shape": f"{M}x{N}x{K}", "flops": flops}
    for epi in ("store", "resid"):
        ms = _time(lambda: op_gemm(A, W, epi, out=out, h32=h32 if epi == "resid" else None), iters)
        res[epi] = {"ms": round(ms, 4), "tflops": round(flops / ms / 1e9, 1)}
    return res


def bench_gemm_fp8(iters):
    M, N, K = 4680, 15360, 5120
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    x = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    wt = (torch.randn(N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    qa = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, device="cuda")
    qw = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty(N, device="cuda")
    op_quantize_e4m3(wt, qw, sw)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ms_q = _time(lambda: op_quantize_e4m3(x, qa, sa), iters)
    ms = _time(lambda: op_gemm_fp8(qa, sa, qw, sw, out), iters)
    flops = 2.0 * M * N * K
    qbytes = M * K * 2 + M * K + M * 4
    return {"mode": "gemm_fp8", "shape": f"{M}x{N}x{K} e4m3", "ms": round(ms, 4),
            "tflops": round(flops / ms / 1e9, 1), "flops": flops,
            "quantize": {"ms": round(ms_q, 4), "gbs": round(qbytes / ms_q / 1e6, 1), "bytes": qbytes}}


def bench_euler(iters):
    rows, C, G = 1 << 20, 64, 4
    x = torch.randn(rows, C, device="cuda")
    v = torch.randn(rows, C, device="cuda")
    dt = [-0.25] * G
    ms = _time(lambda: op_euler(x, v, dt, rows // G), iters)
    nbytes = 3 * rows * C * 4
    return {"mode": "euler", "shape": f"{rows}x{C} fp32", "ms": round(ms, 4), "gbs": round(nbytes / ms / 1e6, 1),
            "bytes": nbytes}


def bench_rerope(iters, layers=8):
    from types import SimpleNamespace
    from .stream import LaStream
    cfg = SimpleNamespace(num_layers=layers, hidden=5120, heads=40, head_dim=128, latent_ch=64, grid_h=30, grid_w=52,
                          frames_per_block=3, sink_frames=1, window_blocks=1, timesteps=(1.0, 0.75, 0.5, 0.25, 0.0),
                          rope_split=(22, 21, 21), pairs=(22, 21, 21), rope_theta=10000.0, sink_mode=0, rolling_rope=1,
                          sink_offset_frames=3, schedule=0, dtype=0)
    D, C, F, T = cfg.hidden, cfg.latent_ch, cfg.grid_h * cfg.grid_w, 3 * cfg.grid_h * cfg.grid_w
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    rnd = lambda *sh: (torch.randn(*sh, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    L = cfg.num_layers
    w = dict(w_qkv=[rnd(3 * D, D) for _ in range(L)], w_out=[rnd(D, D) for _ in range(L)], w_in=rnd(D, C),
             w_head=rnd(C, D))
    s = LaStream(cfg, w)
    s.set_sink(torch.randn(F, C, generator=g, device="cuda"))
    x = torch.randn(T, C, generator=g, device="cuda")
    out = torch.empty(T, C, device="cuda")
    for _ in range(3 + 2 + 3):          # fill: every slot active
        s.step(x, out)
    s.synchronize()
    s.profile(True)
    for _ in range(iters):
        s.step(x, out)
    s.synchronize()
    n, tot = s.profile_read("rope")
    s.profile(False)
    s.close()
    ms = tot / n
    nbytes = L * (F * D * 4 + 4 * F * D * 2)
    return {"mode": "rerope", "shape": f"sink {F} tokens x {D}, {L} layers, 4 slots, one launch a tick",
            "ms": round(ms, 4), "gbs": round(nbytes / ms / 1e6, 1), "bytes": nbytes}


def bench_qkv_stream(iters, fp8=False):
    from types import SimpleNamespace
    from .stream import LaStream
    cfg = SimpleNamespace(num_layers=1, hidden=5120, heads=40, head_dim=128, latent_ch=64, grid_h=30, grid_w=52,
                          frames_per_block=3, sink_frames=1, window_blocks=2, timesteps=(1.0, 0.75, 0.5, 0.25, 0.0),
                          rope_split=(22, 21, 21), pairs=(22, 21, 21), rope_theta=10000.0, sink_mode=0, rolling_rope=1,
                          sink_offset_frames=3, schedule=0, dtype=0, proj_fp8=1 if fp8 else 0)
    D, C, F, T = cfg.hidden, cfg.latent_ch, cfg.grid_h * cfg.grid_w, 3 * cfg.grid_h * cfg.grid_w
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    rnd = lambda *sh: (torch.randn(*sh, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    w = dict(w_qkv=[rnd(3 * D, D)], w_out=[rnd(D, D)], w_in=rnd(D, C), w_head=rnd(C, D))
    s = LaStream(cfg, w)
    s.set_sink(torch.randn(F, C, generator=g, device="cuda"))
    x = torch.randn(T, C, generator=g, device="cuda")
    out = torch.empty(T, C, device="cuda")
    for _ in range(3 + 3 + 3):          # fill: every slot active with a full window
        s.step(x, out)
    s.synchronize()
    s.profile(True)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    n = 0
    while True:                         # at least iters ticks and 1.5 s
        s.step(x, out)
        n += 1
        if n >= iters and n % 10 == 0:
            t1.record()
            t1.synchronize()
            if t0.elapsed_time(t1) >= 1500.0:
                break
    s.synchronize()
    res = {"mode": "qkv_stream", "dtype": "e4m3 operands" if fp8 else "bf16", "ticks": n}
    M = 4 * T
    for kind, N, what in (("qkv_gemm", 3 * D, "QKV + RoPE/ring append"), ("out_gemm", D, "output + residual")):
        cnt, tot = s.profile_read(kind)
        ms = tot / cnt
        flops = 2.0 * M * N * D
        res[kind] = {"shape": f"{M}x{N}x{D}", "epilogue": what, "ms": round(ms, 4),
                     "tflops": round(flops / ms / 1e9, 1), "launches": cnt}
    s.profile(False)
    s.close()
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("mode", choices=["attn", "attn_fp8", "gemm", "gemm_out", "euler", "rerope", "gemm_fp8",
                                     "qkv_stream", "all"])
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--layers", type=int, default=8, help="rerope: sublayers of the stream (one launch covers all)")
    ap.add_argument("--fp8", action="store_true", help="qkv_stream: e4m3 projections")
    args = ap.parse_args()
    modes = ["attn", "attn_fp8", "gemm", "gemm_out", "gemm_fp8", "euler", "rerope"] if args.mode == "all" else [args.mode]
    for m in modes:
        clocks = ClockSampler(torch.cuda.current_device())
        clocks.start()
        r = {"attn": bench_attn, "attn_fp8": bench_attn_fp8, "gemm": bench_gemm, "gemm_out": bench_gemm_out,
             "euler": bench_euler, "rerope": lambda it: bench_rerope(it, args.layers),
             "gemm_fp8": bench_gemm_fp8, "qkv_stream": lambda it: bench_qkv_stream(it, args.fp8)}[m](args.iters)
        r["clocks"] = clocks.stop()
        print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
