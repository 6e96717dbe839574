"""Benchmark of the timestep-forced streaming step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--sweep | --ablation] [--no-tpp]

A step is one tick of the 4-slot grouped stream in steady state: 4 in-flight
blocks (one per timestep slot, every window full) through 8 attention
sublayers, the velocity head and the Euler update; each tick finishes one
3-latent-frame block.  value = latent frames/s over all ranks (each rank runs
an independent stream: replicas, weak scaling).  Inputs (weights 1.7 GB, ring
caches 9.2 GB) are larger than L2.  Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle on bounded query-row samples of
the same workload (rank 0 only) and prints the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from streaming_causal_video_timestep_b200.clocks import ClockSampler  # noqa: E402

METRIC = "latent frames/s (4-step stream, 1 B200); attention % of bf16 tensor-core peak"
UNIT = "latent frames/s"
WORKLOAD = dict(
    workload="4-step timestep-forced stream: 4 in-flight blocks x 8 attention sublayers, grouped launch",
    hidden=5120, heads=40, head_dim=128, latent_ch=64, grid="30x52", tokens_per_block=4680, sink_tokens=1560,
    window_blocks=2, keys_per_query=15600, timesteps=[1.0, 0.75, 0.5, 0.25, 0.0], layers=8,
    dtype="bf16 weights, activations and attention operands (q pre-scaled); fp32 accumulate, residual stream and latent",
    l2="inputs larger than L2: 1.68 GB weights + 9.2 GB ring caches read per tick",
    data="synthetic: N(0,1) latents, N(0,0.02) weights, seeded")


# DRAM bytes (read + write) of one slot's attention launch (4680 queries x 15,600 keys x 40 heads x 128,
# bf16 q/K/V and output) from one ncu capture of the one-slot attention microbenchmark of the kernel with
# the warp-wide MMA issuer and 2 of 8 exponential pairs on the FMA pipe: 385.2 MB read + 43.3 MB written,
# against 415.2 MB of algorithmic bytes.  The grouped launch of the stream reads the disjoint q / K / V of
# its S slots, so its traffic is S times this.
ATTN_DRAM_BYTES_PER_SLOT = 428.5e6
# FFN width of the full DiT block in the ablation: the 14B Wan-style DiT's 13824 (2.7 x 5120)
DIT_FFN = 13824
# Audio of a block for the DiT block's cross-attention (synthetic sizes; the pages give none):
# 256 tokens of width 1024
DIT_AUDIO = (256, 1024)


def max_over_ranks(x, device):
    """The largest of every rank's x (the job's time is its slowest rank's); x itself on one rank."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(frames_per_tick, ticks, world, seconds):
    """Whole-job latent frames/s: every rank runs `ticks` ticks of its own stream (weak scaling)."""
    return frames_per_tick * ticks * world / seconds


def _attn_flops_per_slot(T, F, nw, H, d):
    nk = F + nw * T + T
    return 4.0 * T * nk * d * H


def kernel_entries(kinds, steps, L, S, T, D, C, F, attn_tflops, pk):
    """Per-kernel-kind figures of the timed ticks: kinds maps a kind to (launches,
    total ms) from the library's profiling counters.  Tensor-core kinds get
    TFLOP/s and the fraction of the measured sustained bf16 peak; the sink
    re-rope gets GB/s and the fraction of the measured HBM copy."""
    gemm_flops = {"qkv_gemm": 2.0 * S * T * D * 3 * D, "out_gemm": 2.0 * S * T * D * D,
                  "in_proj": 2.0 * S * T * C * D, "head": 2.0 * S * T * D * C}
    kernels = {}
    for kind, (n, tot) in kinds.items():
        if n == 0:
            continue
        avg = tot / n
        e = {"launches": n, "ms_avg": round(avg, 4), "ms_per_step": round(tot / steps, 3)}
        if kind == "attn":
            e["tflops"] = round(attn_tflops, 1)
        elif kind == "rope":
            # sink re-rope of every active slot: read each layer's fp32 un-roped sink K once,
            # write S bf16 roped copies (the block's RoPE + append is fused into the QKV GEMM);
            # one launch covers all L layers of a pass (L steps / n layers a launch)
            layers = max(1, round(L * steps / n))
            nbytes = layers * (F * D * 4 + S * F * D * 2)
            e["gbs"] = round(nbytes / (avg / 1000.0) / 1e9, 1)
            e["frac_hbm"] = round(e["gbs"] / pk["hbm"], 3)
            e["bytes_per_launch"] = nbytes
        elif kind in gemm_flops and n >= steps * (L if kind in ("qkv_gemm", "out_gemm") else 1):
            e["tflops"] = round(gemm_flops[kind] / (avg / 1000.0) / 1e12, 1)
        if "tflops" in e:
            e["frac_sustained"] = round(e["tflops"] / pk["tflops_sust"], 3)
        kernels[kind] = e
    return kernels


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(tflops=j["bf16_tflops"], tflops_sust=j["bf16_tflops_sustained"], hbm=j["hbm_gbs"],
                    src="measured")
    return dict(tflops=1590.0, tflops_sust=1400.0, hbm=6650.0, src="fallback")


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def append_marginal(s, xs, x_out, S, T, D, ticks=6):
    """The Rolling RoPE + ring append runs as the epilogue of the QKV GEMM.  Its
    cost is the difference between that GEMM (all S slots' rows, M = S T, N = 3D,
    K = D), timed by the stream's counters, and a plain bf16 store of the same
    GEMM shape launched between the stream's ticks, so that both run in the
    same clock regime (a power-capped GPU clocks a long GEMM-only loop lower
    than the mixed stream).  Against it stand the bytes a separate RoPE + append
    kernel would move (read qkv, write q, K and V: 2 x M x 3D x 2 B)."""
    import torch
    from streaming_causal_video_timestep_b200 import op_gemm

    M, N, K = S * T, 3 * D, D
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    A = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    op_gemm(A, W, "store", out=out)
    torch.cuda.synchronize()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    s.profile(True)
    evs = []
    for k in range(ticks):
        s.step(xs[k % len(xs)], x_out)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s.stream)
        op_gemm(A, W, "store", out=out, stream=s.stream)
        e1.record(s.stream)
        evs.append((e0, e1))
    s.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    n, tot = s.profile_read("qkv_gemm")
    s.profile(False)
    ms_epi = tot / max(n, 1)
    ms_plain = sum(a.elapsed_time(b_) for a, b_ in evs) / len(evs)
    standalone = 2 * M * N * 2
    marginal = ms_epi - ms_plain
    del A, W, out
    torch.cuda.empty_cache()
    return {"qkv_gemm_with_rope_append_ms": round(ms_epi, 4), "qkv_gemm_plain_store_ms": round(ms_plain, 4),
            "marginal_ms": round(marginal, 4), "marginal_frac_of_gemm": round(marginal / ms_epi, 4),
            "standalone_bytes": standalone,
            "standalone_ms_at_measured_hbm": round(standalone / (_peaks()["hbm"] * 1e9) * 1e3, 4),
            "shape": f"{M}x{N}x{K}", "ticks": ticks, "clocks": clk,
            "note": "plain-store GEMM launched between the stream's ticks (same clock regime); the epilogue "
                    "writes as many bytes as the plain store (q, K, V vs qkv); a separate RoPE + append kernel "
                    "would move standalone_bytes"}


def run_gpu(args, rank, world, local_rank):
    import torch
    from streaming_causal_video_timestep_b200 import LaStream
    from workloads import STREAM

    torch.cuda.set_device(local_rank)
    wl = STREAM
    cfg = wl.cfg
    T, C, D, F, H, d = cfg.block_tokens, cfg.latent_ch, cfg.hidden, cfg.frame_tokens, cfg.heads, cfg.head_dim
    S, nw, L = cfg.num_steps, cfg.window_blocks, cfg.num_layers
    g = torch.Generator(device="cuda")
    g.manual_seed(1000 + rank)
    bf = torch.bfloat16

    def rnd(shape, std):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(bf)

    weights = dict(w_qkv=[rnd((3 * D, D), wl.w_std) for _ in range(L)],
                   w_out=[rnd((D, D), wl.w_std) for _ in range(L)],
                   w_in=rnd((D, C), 1.0 / C ** 0.5), w_head=rnd((C, D), wl.head_std))
    s = LaStream(cfg, weights)
    s.set_sink(torch.randn((F, C), generator=g, device="cuda"))
    xs = [torch.randn((T, C), generator=g, device="cuda") for _ in range(4)]
    x_out = torch.empty((T, C), device="cuda")
    fill = (S - 1) + nw + 1          # every slot active with a full window from here on
    k = 0
    ph = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ph[0].record()
    for _ in range(fill + args.warmup):
        fin = s.step(xs[k % 4], x_out)
        k += 1
        if k == S:                   # block 0 leaves the last slot at tick S - 1
            ph[1].record()
            assert fin == 0
        if k == fill:
            ph[2].record()
    s.synchronize()
    torch.cuda.synchronize()
    first_block_ms, fill_ms = ph[0].elapsed_time(ph[1]), ph[0].elapsed_time(ph[2])
    st = s.index_state()
    per = 8 + 3 * cfg.ring_entries
    assert all(st[4 + i * per] >= nw for i in range(S)), "not in steady state"

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    launches0 = s.launch_count()
    s.profile(True)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        s.step(xs[k % 4], x_out)
        k += 1
    ev1.record(stream)
    s.synchronize()
    torch.cuda.synchronize()
    launches = s.launch_count() - launches0
    ms = ev0.elapsed_time(ev1)
    kinds = {kind: s.profile_read(kind) for kind in ("in_proj", "qkv_gemm", "rope", "attn", "out_gemm", "head",
                                                     "other")}
    s.profile(False)
    clk = clocks.stop()
    ms = max_over_ranks(ms, "cuda")
    if dist:
        tdist.barrier()

    # end to end through the public host-buffer call: every tick copies its new
    # block from pinned host memory and its finished block back to pinned host
    # memory inside the timed region.  Two output buffers: the host enqueues tick
    # i, then waits for tick i - 1 and reads its block, so host work overlaps
    # the GPU the way a streaming server runs.
    xh = [torch.randn((T, C)).pin_memory() for _ in range(2)]
    oh = [torch.empty((T, C)).pin_memory() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    for _ in range(2):
        s.step_host(xh[0], oh[0])
    s.synchronize()
    if dist:
        tdist.barrier()
    e2e_steps = max(3, min(args.steps, 10))
    read_back = 0.0
    t0 = time.perf_counter()
    for i in range(e2e_steps):
        fin = s.step_host(xh[i % 2], oh[i % 2])
        done[i % 2].record(s.stream)
        assert fin >= 0
        if i > 0:
            done[(i - 1) % 2].synchronize()
            read_back += float(oh[(i - 1) % 2][0, 0])
    done[(e2e_steps - 1) % 2].synchronize()
    read_back += float(oh[(e2e_steps - 1) % 2][0, 0])
    s.synchronize()
    e2e_s = time.perf_counter() - t0
    assert read_back == read_back, "NaN in the latents read back"
    e2e_s = max_over_ranks(e2e_s, "cuda")
    # drain: S - 1 ticks without new blocks finish the blocks still in flight
    dr = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    dr[0].record()
    for _ in range(S - 1):
        assert s.step(None, x_out) >= 0
    dr[1].record()
    torch.cuda.synchronize()
    drain_ms = dr[0].elapsed_time(dr[1])
    # refill the pipeline, then the append's marginal cost between ticks
    for _ in range(fill):
        s.step(xs[k % 4], x_out)
        k += 1
    append = append_marginal(s, xs, x_out, S, T, D)
    s.close()
    del s, weights
    torch.cuda.empty_cache()

    frames_per_tick = cfg.frames_per_block
    value = job_throughput(frames_per_tick, args.steps, world, ms / 1000.0)
    e2e_value = job_throughput(frames_per_tick, e2e_steps, world, e2e_s)
    pk = _peaks()
    n_attn, ms_attn = kinds["attn"]
    attn_flops_launch = S * _attn_flops_per_slot(T, F, nw, H, d)
    attn_ms_avg = ms_attn / max(n_attn, 1)
    achieved = attn_flops_launch / (attn_ms_avg / 1000.0) / 1e12
    peak = pk["tflops_sust"]
    kernels = kernel_entries(kinds, args.steps, L, S, T, D, C, F, achieved, pk)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"replicas x{world} (independent streams, no collective)"),
        "roofline": {"bound": "tensor", "kernel": "block-causal attention (tcgen05)", "achieved": round(achieved, 1),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": ATTN_DRAM_BYTES_PER_SLOT * S,
                     "traffic_unit": "bytes per launch (ncu dram read+write, one-slot capture x slots)",
                     "peak_source": f"{pk['src']} bf16 sustained (the kernel's operands are bf16)",
                     "algorithmic_flops_per_launch": attn_flops_launch},
        "kernels": kernels,
        "gpu_launches": int(launches),
        "phases": {"first_finished_block_ms": round(first_block_ms, 3), "fill_ticks": fill,
                   "fill_ms": round(fill_ms, 3), "drain_ticks": S - 1, "drain_ms": round(drain_ms, 3),
                   "note": "rank 0; fill = ticks until every slot is active with a full window (untimed by value)"},
        "clocks": clk,
        "append": append,
        "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": T * C * 4,
                "d2h_bytes_per_step": T * C * 4, "steps": e2e_steps},
    }
    return line


def run_tpp(args, rank, world, local_rank):
    """The timestep pipeline across GPUs (the pages' TPP): world / num_steps
    pipelines of num_steps consecutive ranks; rank r of a pipeline owns denoising
    step r of every block with its own cache (an LA_SCHED_SLOT stream of the
    headline workload) and hands the latent to rank r + 1 by NCCL send/recv (no
    other data path; the Adaptive Attention Sink is broadcast once).  Every rank
    runs this; rank 0 returns the record.  Timed on the device: K ticks between
    CUDA events on each rank, max over all ranks."""
    import torch
    import torch.distributed as tdist
    from streaming_causal_video_timestep_b200 import LaStream
    from streaming_causal_video_timestep_b200.tpp import DistTransport, TppRank
    from workloads import SCHED_SLOT, SINK_AAS, STREAM

    wl = STREAM
    S = wl.cfg.num_steps
    G = world // S
    groups = [tdist.new_group(list(range(p * S, (p + 1) * S))) for p in range(G)]
    pid, r = rank // S, rank % S
    cfg = wl.cfg.replace(schedule=SCHED_SLOT, slot_index=r)
    T, C, D, F = cfg.block_tokens, cfg.latent_ch, cfg.hidden, cfg.frame_tokens
    L = cfg.num_layers
    dev = torch.device("cuda", local_rank)
    g = torch.Generator(device="cuda")
    g.manual_seed(2000 + pid)               # the ranks of a pipeline hold the same model and sink
    bf = torch.bfloat16
    rnd = lambda shape, std: (torch.randn(shape, generator=g, device="cuda") * std).to(bf)
    weights = dict(w_qkv=[rnd((3 * D, D), wl.w_std) for _ in range(L)],
                   w_out=[rnd((D, D), wl.w_std) for _ in range(L)],
                   w_in=rnd((D, C), 1.0 / C ** 0.5), w_head=rnd((C, D), wl.head_std))
    s = LaStream(cfg, weights)
    s.set_sink(torch.randn((F, C), generator=g, device="cuda"))
    xs = [torch.randn((T, C), generator=g, device="cuda") for _ in range(4)]
    tr = DistTransport(r, S, dev, group=groups[pid], base=pid * S)
    me = TppRank(s, r, S, tr, dev, S, cfg.sink_tokens, cfg.sink_mode == SINK_AAS)
    k = 0

    def tick():
        nonlocal k
        fin = me.tick(xs[k % 4] if r == 0 else None)
        k += 1
        return fin[0]

    tdist.barrier()
    torch.cuda.synchronize()
    ev_first = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev_first[0].record()
    first_ms = 0.0
    for _ in range(S - 1 + args.warmup):     # fill: block 0 leaves the last rank at tick S - 1
        if tick() == 0:
            ev_first[1].record()
    torch.cuda.synchronize()
    if r == S - 1:
        first_ms = ev_first[0].elapsed_time(ev_first[1])
    tdist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        tick()
    ev[1].record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = max_over_ranks(ev[0].elapsed_time(ev[1]), "cuda")
    first_ms = max_over_ranks(first_ms, "cuda")
    me.close()                               # the last tick's hand-off is received before the next test
    # the hand-off alone: the message a rank sends each tick (block id + T x C fp32),
    # rank r -> r + 1 of every pipeline at once, timed on each rank, max over ranks
    msg = [torch.zeros(1, dtype=torch.int64, device=dev), torch.zeros((T, C), dtype=torch.float32, device=dev)]
    layout = [(tuple(t.shape), t.dtype) for t in msg]
    tdist.barrier()
    torch.cuda.synchronize()
    hev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = 20
    hev[0].record()
    for _ in range(reps):
        # the pipeline's own exchange: one batched send / receive a rank
        tr.exchange(msg if r < S - 1 else None, layout if r > 0 else None)
    hev[1].record()
    torch.cuda.synchronize()
    hand_ms = max_over_ranks(hev[0].elapsed_time(hev[1]) / reps, "cuda")
    tdist.barrier()
    s.close()
    del s, weights
    torch.cuda.empty_cache()
    for grp in groups:
        tdist.destroy_process_group(grp)
    return {"pipelines": G, "ranks_per_pipeline": S,
            "latent_frames_per_s": round(job_throughput(cfg.frames_per_block, args.steps, G, ms / 1000.0), 3),
            "ms_per_tick": round(ms / args.steps, 3), "steps": args.steps,
            "first_finished_block_ms": round(first_ms, 3),
            "handoff_bytes_per_tick_per_link": 8 + T * C * 4, "handoff_ms": round(hand_ms, 4),
            "clocks": clk,
            "note": "rank r of each pipeline owns step r with its own cache (LA_SCHED_SLOT stream); NCCL "
                    "send/recv of the latent between consecutive ranks; the AAS sink broadcast once"}


# ---------------------------------------------------------------------------
# the oracle on the host: bounded query-row samples of one slot's sublayer
# ---------------------------------------------------------------------------
class OracleSample:
    """One attention sublayer of one slot in steady state (window full), for a
    sample of the block's query rows, with the oracle's own functions: QKV
    projection, 3D Rolling RoPE, block-causal attention over sink + 2 window
    blocks + the block (15,600 keys), output projection.  Per-row work is the
    same for every row, so time x (rows of a block / sampled rows) x (slots x
    layers) estimates one tick."""

    def __init__(self, rows):
        import numpy as np
        from oracle.rope import block_positions, sink_positions
        from workloads import STREAM
        self.np = np
        c = STREAM.cfg
        self.c = c
        self.rows = rows
        T, D, H, d, F = c.block_tokens, c.hidden, c.heads, c.head_dim, c.frame_tokens
        rng = np.random.default_rng(7)
        self.w_qkv = rng.standard_normal((3 * D, D)) * 0.02
        self.w_out = rng.standard_normal((D, D)) * 0.02
        self.h = rng.standard_normal((rows, D))
        self.b = 2
        self.blocks = {b: (rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d))) for b in (0, 1)}
        self.self_v = rng.standard_normal((T, H, d))
        self.self_k = rng.standard_normal((T, H, d))
        self.sink = (rng.standard_normal((F, H, d)), rng.standard_normal((F, H, d)))
        self.pos = block_positions(c, self.b)
        self.spos = sink_positions(c, 3 * self.b - 3)

    def step(self):
        from oracle import block_causal_attention, rope_rotate
        c, r = self.c, self.rows
        D, H, d = c.hidden, c.heads, c.head_dim
        qkv = self.h @ self.w_qkv.T
        q = qkv[:, :D].reshape(r, H, d)
        k = qkv[:, D:2 * D].reshape(r, H, d)
        pt, ph, pw = (p[:r] for p in self.pos)
        qr = rope_rotate(q, pt, ph, pw, c.pairs, c.rope_theta)
        kr = rope_rotate(k, pt, ph, pw, c.pairs, c.rope_theta)
        self.self_k[:r] = kr
        blocks = dict(self.blocks)
        blocks[self.b] = (self.self_k, self.self_v)
        sk = rope_rotate(self.sink[0], *self.spos, c.pairs, c.rope_theta)
        o = block_causal_attention(qr, blocks, (sk, self.sink[1]), qblock=self.b, window=c.window_blocks)
        return self.h + o.reshape(r, D) @ self.w_out.T

    def frames_per_s(self, seconds_per_step):
        c = self.c
        tick_s = seconds_per_step * (c.block_tokens / self.rows) * c.num_steps * c.num_layers
        return c.frames_per_block / tick_s


def cpu_baseline(rows=1560, reps=1):
    """The oracle as it stands on this host's cores: one sublayer of one slot for
    `rows` of the block's 4680 query rows (about 10 s at 1560 rows on 16 cores),
    scaled to a tick."""
    smp = OracleSample(rows)
    t0 = time.perf_counter()
    for _ in range(reps):
        smp.step()
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(smp.frames_per_s(dt), 6), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
            "sample": (f"1 sublayer, 1 slot, {rows}/4680 rows x 15600 keys, {dt:.1f} s; "
                       f"x{4680 / rows:.0f} rows x4 slots x8 layers")}


def run_sweep(args):
    """One JSON line per shape-sweep point (two token grids x cache windows 1, 2, 4, 8; one attention
    sublayer; 4 slots as one grouped launch) and one for the standalone Euler update.  Not the
    headline metric: each point reports the attention kernel's TFLOP/s and the sink re-rope's GB/s
    against the measured peaks."""
    import torch
    from streaming_causal_video_timestep_b200 import LaStream, op_euler
    from workloads import SWEEP

    torch.cuda.set_device(0)
    pk = _peaks()
    bf = torch.bfloat16
    for wl in SWEEP:
        cfg = wl.cfg
        T, C, D, F, H, d = cfg.block_tokens, cfg.latent_ch, cfg.hidden, cfg.frame_tokens, cfg.heads, cfg.head_dim
        S, nw, L = cfg.num_steps, cfg.window_blocks, cfg.num_layers
        g = torch.Generator(device="cuda")
        g.manual_seed(wl.seed)
        rnd = lambda shape, std: (torch.randn(shape, generator=g, device="cuda") * std).to(bf)
        weights = dict(w_qkv=[rnd((3 * D, D), wl.w_std) for _ in range(L)],
                       w_out=[rnd((D, D), wl.w_std) for _ in range(L)],
                       w_in=rnd((D, C), 1.0 / C ** 0.5), w_head=rnd((C, D), wl.head_std))
        s = LaStream(cfg, weights)
        s.set_sink(torch.randn((F, C), generator=g, device="cuda"))
        xs = [torch.randn((T, C), generator=g, device="cuda") for _ in range(2)]
        x_out = torch.empty((T, C), device="cuda")
        clocks = ClockSampler(0)
        clocks.start()
        for k in range((S - 1) + nw + 1 + args.warmup):
            s.step(xs[k % 2], x_out)
        s.synchronize()
        s.profile(True)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for k in range(args.steps):
            s.step(xs[k % 2], x_out)
        ev1.record()
        s.synchronize()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / args.steps
        clk = clocks.stop()
        n_a, t_a = s.profile_read("attn")
        n_r, t_r = s.profile_read("rope")
        s.profile(False)
        attn_flops = S * _attn_flops_per_slot(T, F, nw, H, d)
        attn_tf = attn_flops / (t_a / n_a / 1000.0) / 1e12
        rope_bytes = F * D * 4 + S * F * D * 2
        rope_gbs = rope_bytes / (t_r / n_r / 1000.0) / 1e9
        print(json.dumps({"sweep": wl.name, "grid": f"{cfg.grid_h}x{cfg.grid_w}", "window_blocks": nw,
                          "keys_per_query": F + nw * T + T, "ms_per_tick": round(ms, 3),
                          "latent_frames_per_s": round(cfg.frames_per_block / (ms / 1000.0), 2),
                          "attn": {"tflops": round(attn_tf, 1), "flops_per_launch": attn_flops,
                                   "frac_sustained": round(attn_tf / pk["tflops_sust"], 3),
                                   "frac_burst": round(attn_tf / pk["tflops"], 3),
                                   "frac_spec_2250": round(attn_tf / 2250.0, 3)},
                          "sink_rerope": {"gbs": round(rope_gbs, 1), "bytes_per_launch": rope_bytes,
                                          "frac_hbm": round(rope_gbs / pk["hbm"], 3)},
                          "peaks": pk["src"], "clocks": clk}), flush=True)
        s.close()
        del s, weights
        torch.cuda.empty_cache()
    rows, C, G = 1 << 20, 64, 4   # 256 MB per tensor, larger than L2
    x = torch.randn(rows, C, device="cuda")
    v = torch.randn(rows, C, device="cuda")
    clocks = ClockSampler(0)
    clocks.start()
    for _ in range(args.warmup):
        op_euler(x, v, [-0.25] * G, rows // G)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_euler = max(args.steps, 2000)     # ~0.25 ms a launch: enough launches to cover clock samples
    ev0.record()
    for _ in range(n_euler):
        op_euler(x, v, [-0.25] * G, rows // G)
    ev1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / n_euler
    gbs = 3 * rows * C * 4 / (ms / 1000.0) / 1e9
    print(json.dumps({"sweep": "euler_standalone", "shape": f"{rows}x{C} fp32, {G} timestep groups",
                      "ms": round(ms, 4), "gbs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm"], 3),
                      "note": "in the stream the Euler update is fused into the velocity-head GEMM epilogue",
                      "clocks": clk}),
          flush=True)


def run_ablation(args):
    """Seconds per block at the headline shape (8 sublayers, 14B-like, window 2) for the
    schedules the pages compare (papernotes note, inference-efficiency ablation, the paper's Table 3): the grouped timestep-forced stream
    (4 blocks in flight, NFE 4), the same cache sequentially (one block through its 4 steps per
    call, NFE 4), and the clean-cache refresh the method removes (4 steps + 1 refresh forward,
    NFE 5); the e4m3 rows of the operator-optimisation row; and the fixed-noise cache the
    key findings compare (the paper's Table 6; same kernels and NFE as the sequential row).
    One JSON line each."""
    import torch
    from streaming_causal_video_timestep_b200 import LaStream
    from workloads import (BLOCK_ATTN, BLOCK_DIT, CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP, CACHE_TIMESTEP,
                           SCHED_PIPELINED, SCHED_SEQUENTIAL, STREAM)

    torch.cuda.set_device(0)
    bf = torch.bfloat16
    only = set(args.ablation_rows.split(",")) if args.ablation_rows else None
    rows = (("timestep-forced, grouped pipeline", SCHED_PIPELINED, CACHE_TIMESTEP, 4, 0, 0, 0),
            ("timestep-forced, sequential", SCHED_SEQUENTIAL, CACHE_TIMESTEP, 4, 0, 0, 0),
            ("clean-cache refresh, sequential", SCHED_SEQUENTIAL, CACHE_CLEAN_REFRESH, 5, 0, 0, 0),
            ("timestep-forced, grouped pipeline, e4m3 projections", SCHED_PIPELINED, CACHE_TIMESTEP, 4, 1, 0, 0),
            ("timestep-forced, grouped pipeline, e4m3 attention", SCHED_PIPELINED, CACHE_TIMESTEP, 4, 0, 1, 0),
            ("timestep-forced, grouped pipeline, e4m3 projections and attention", SCHED_PIPELINED,
             CACHE_TIMESTEP, 4, 1, 1, 0),
            ("fixed-noise cache (prior blocks at the last step's noise), sequential", SCHED_SEQUENTIAL,
             CACHE_FIXED_STEP, 4, 0, 0, 0),
            ("timestep-forced, grouped pipeline, full DiT block (AdaLN, GELU FFN 13824)", SCHED_PIPELINED,
             CACHE_TIMESTEP, 4, 0, 0, DIT_FFN),
            ("timestep-forced, grouped pipeline, full DiT block with audio cross-attention (256 x 1024)",
             SCHED_PIPELINED, CACHE_TIMESTEP, 4, 0, 0, -DIT_FFN))
    for idx, (name, sched, mode, nfe, fp8, afp8, ffn) in enumerate(rows):
        if only is not None and str(idx) not in only:
            continue
        audio = ffn < 0            # a negative FFN width marks the row with the audio cross-attention
        ffn = abs(ffn)
        cfg = STREAM.cfg.replace(schedule=sched, cache_mode=mode, proj_fp8=fp8, attn_fp8=afp8,
                                 cache_step=STREAM.cfg.num_steps - 1,
                                 block_kind=BLOCK_DIT if ffn else BLOCK_ATTN, ffn_dim=ffn,
                                 audio_tokens=DIT_AUDIO[0] if audio else 0, audio_dim=DIT_AUDIO[1] if audio else 0)
        T, C, D, F = cfg.block_tokens, cfg.latent_ch, cfg.hidden, cfg.frame_tokens
        S, nw, L = cfg.num_steps, cfg.window_blocks, cfg.num_layers
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        rnd = lambda shape, std: (torch.randn(shape, generator=g, device="cuda") * std).to(bf)
        weights = dict(w_qkv=[rnd((3 * D, D), STREAM.w_std) for _ in range(L)],
                       w_out=[rnd((D, D), STREAM.w_std) for _ in range(L)],
                       w_in=rnd((D, C), 1.0 / C ** 0.5), w_head=rnd((C, D), STREAM.head_std))
        if ffn:
            # the DiT block: FFN weights and the AdaLN table (shifts, scales ~ N(0, 0.1^2), gates ~ N(1, 0.1^2))
            weights["w_ffn1"] = [rnd((ffn, D), STREAM.w_std) for _ in range(L)]
            weights["w_ffn2"] = [rnd((D, ffn), STREAM.w_std) for _ in range(L)]
            ada = torch.randn((L, S + 1, 6, D), generator=g, device="cuda") * 0.1
            ada[:, :, 2] += 1.0
            ada[:, :, 5] += 1.0
            weights["ada"] = ada.contiguous()
        if audio:
            weights["w_qc"] = [rnd((D, D), STREAM.w_std) for _ in range(L)]
            weights["w_kvc"] = [rnd((2 * D, DIT_AUDIO[1]), DIT_AUDIO[1] ** -0.5) for _ in range(L)]
            weights["w_oc"] = [rnd((D, D), STREAM.w_std) for _ in range(L)]
        aud = torch.randn(DIT_AUDIO, generator=g, device="cuda") if audio else None
        s = LaStream(cfg, weights)
        s.set_sink(torch.randn((F, C), generator=g, device="cuda"))
        xs = [torch.randn((T, C), generator=g, device="cuda") for _ in range(2)]
        x_out = torch.empty((T, C), device="cuda")
        fill = ((S - 1) if sched == SCHED_PIPELINED else 0) + nw + 1 + args.warmup
        clocks = ClockSampler(0)
        clocks.start()
        for k in range(fill):
            s.step(xs[k % 2], x_out, audio=aud)
        s.synchronize()
        s.profile(True)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for k in range(args.steps):
            assert s.step(xs[k % 2], x_out, audio=aud) >= 0
        ev1.record()
        s.synchronize()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / args.steps
        clk = clocks.stop()
        kinds = {kd: round(s.profile_read(kd)[1] / args.steps, 3)
                 for kd in ("qkv_gemm", "attn", "out_gemm", "other") + (("ffn",) if ffn else ())
                 + (("cross",) if audio else ())}
        extra = {}
        if ffn:
            # per call (a tick, or a block's S steps): S passes x L layers x two GEMMs of 2 T D F flops
            ffn_flops = 4.0 * T * D * ffn * L * S
            extra["ffn_tflops"] = round(ffn_flops / (kinds["ffn"] / 1000.0) / 1e12, 1)
        s.profile(False)
        print(json.dumps({"ablation": name, "nfe_per_block": nfe, "ms_per_block": round(ms, 3),
                          "latent_frames_per_s": round(cfg.frames_per_block / (ms / 1000.0), 3),
                          "ms_per_block_by_kind": kinds, **extra,
                          "config": ("8 DiT blocks (AdaLN, GELU FFN %d%s)" % (
                                         ffn, ", audio cross-attention %d x %d" % DIT_AUDIO if audio else "")
                                     if ffn else "8 sublayers")
                                    + ", hidden 5120, 40x128 heads, 30x52 grid, window 2, "
                                    + ", ".join([x for x in ("e4m3 QKV/output projections" if fp8 else "",
                                                             "e4m3 attention" if afp8 else "") if x]
                                                or ["bf16"]),
                          "clocks": clk}),
              flush=True)
        s.close()
        del s, weights
        torch.cuda.empty_cache()


def run_reference(args):
    smp = OracleSample(rows=234)
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    dt = (time.perf_counter() - t0) / args.steps
    v = smp.frames_per_s(dt)
    sample = f"per step: 1 sublayer, 1 slot, 234/4680 rows, {dt:.2f} s; x20 rows x4 slots x8 layers"
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1000.0, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(WORKLOAD),
            "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="shape sweep lines instead of the headline line")
    ap.add_argument("--ablation", action="store_true",
                    help="seconds per block: grouped pipeline vs sequential vs clean-cache refresh")
    ap.add_argument("--ablation-rows", default="",
                    help="comma-separated row indices of --ablation to run (default: all)")
    ap.add_argument("--no-tpp", action="store_true",
                    help="with N a multiple of the step count, skip the timestep-pipeline sub-record")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return
    if args.ablation:
        if rank == 0:
            run_ablation(args)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        # a collective that times out aborts its communicator and raises in the waiting
        # call (instead of tearing the process down), so rank 0 can still print its line
        os.environ.setdefault("TORCH_NCCL_ASYNC_ERROR_HANDLING", "2")
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    line = run_gpu(args, rank, world, local_rank)
    from workloads import STREAM
    if world > 1 and world % STREAM.cfg.num_steps == 0 and not args.no_tpp:
        # the pipeline arm must not cost the replicas line: an error in it (or a rank
        # that times out in one of its collectives) is reported in the record instead
        try:
            tpp = run_tpp(args, rank, world, local_rank)
        except Exception as e:       # noqa: BLE001 - any failure of the sub-record
            tpp = {"error": f"{type(e).__name__}: {e}"[:300]}
        if rank == 0:
            line["tpp"] = tpp
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
