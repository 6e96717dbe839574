"""Stream configurations and seeded synthetic inputs.

This module is shared by the CUDA path's tests/bench and by the fp64 oracle.
It holds shapes, flags and random-number draws only: none of the method's
arithmetic (projection, RoPE, attention, Euler) lives here.

The shapes follow the Live Avatar pages (arXiv 2512.04677):
  * 3 latent frames per autoregressive block (papernotes ECCV2026 note,
    "整体框架" / overall framework);
  * one sink frame, a rolling KV window of N prior blocks per timestep slot
    (gitcode study blog, question 1 table);
  * 4 distilled timesteps (10100.com article, summary; papernotes Table 3, NFE 4).
The timestep values, the 14B-like widths and the weight distributions are not
on the pages; they are the workload definitions of this repository.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

SINK_FIXED = 0
SINK_AAS = 1
SCHED_PIPELINED = 0
SCHED_SEQUENTIAL = 1
SCHED_SLOT = 2             # one rank of the timestep pipeline across GPUs: step slot_index of each block
DTYPE_BF16 = 0
DTYPE_FP32 = 1
CACHE_TIMESTEP = 0         # noisy K/V of each step in that step's own cache (timestep forcing)
CACHE_CLEAN_REFRESH = 1    # one cache of clean K/V, refreshed by an extra forward of x0 per block (NFE S+1)
CACHE_FIXED_STEP = 2       # every step reads the prior blocks' K/V of one fixed step (cache_step): fixed noise
BLOCK_ATTN = 0             # each layer: the attention sublayer of the step
BLOCK_DIT = 1              # each layer: a full DiT block (AdaLN-modulated attention and GELU FFN sub-blocks)


def default_rope_split(head_dim: int) -> tuple:
    """Rotary pairs per axis (t, h, w): p_h = p_w = floor(P/3), p_t = rest, P = d/2."""
    p = head_dim // 2
    ph = p // 3
    return (p - 2 * ph, ph, ph)


@dataclass(frozen=True)
class StreamConfig:
    num_layers: int
    hidden: int
    heads: int
    head_dim: int
    latent_ch: int
    grid_h: int
    grid_w: int
    frames_per_block: int = 3
    sink_frames: int = 1
    window_blocks: int = 2
    # num_steps + 1 values, strictly descending; the last one is the end time.
    timesteps: tuple = (1.0, 0.75, 0.5, 0.25, 0.0)
    rope_split: Optional[tuple] = None      # rotary PAIRS (t, h, w); None -> default rule
    rope_theta: float = 10000.0
    sink_mode: int = SINK_AAS
    rolling_rope: int = 1
    sink_offset_frames: int = 3
    schedule: int = SCHED_PIPELINED
    dtype: int = DTYPE_BF16
    cache_mode: int = CACHE_TIMESTEP
    proj_fp8: int = 0        # 1: QKV / output projections on per-row-quantized e4m3 operands (bf16 streams)
    attn_fp8: int = 0        # 1: the denoising passes' attention on e4m3 q / K / V (bf16 streams, head_dim 128)
    cache_step: int = 0      # CACHE_FIXED_STEP: the step whose K/V every step reads for the prior blocks
    block_kind: int = BLOCK_ATTN
    ffn_dim: int = 0         # BLOCK_DIT: hidden width of the FFN
    audio_tokens: int = 0    # BLOCK_DIT: audio tokens per block for the cross-attention (0: none)
    audio_dim: int = 0       # their feature width
    slot_index: int = 0      # SCHED_SLOT: the step this rank runs

    @property
    def num_steps(self) -> int:
        return len(self.timesteps) - 1

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def block_tokens(self) -> int:
        return self.frames_per_block * self.frame_tokens

    @property
    def sink_tokens(self) -> int:
        return self.sink_frames * self.frame_tokens

    @property
    def ring_entries(self) -> int:
        return self.window_blocks + 1

    @property
    def pairs(self) -> tuple:
        return tuple(self.rope_split) if self.rope_split is not None else default_rope_split(self.head_dim)

    @property
    def identity_in(self) -> bool:
        return self.latent_ch == self.hidden

    def replace(self, **kw) -> "StreamConfig":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: StreamConfig
    seed: int
    num_blocks: int
    w_std: float            # std of the QKV / output projection weights
    head_std: float = 0.02  # std of the velocity head (latent_ch != hidden only)
    fresh_step_inputs: bool = False   # every (block, step) input is fresh noise
    description: str = ""


# ---------------------------------------------------------------------------
# The five workloads.
# ---------------------------------------------------------------------------
TINY = Workload(
    name="tiny-fp32",
    cfg=StreamConfig(num_layers=1, hidden=64, heads=1, head_dim=64, latent_ch=64,
                     grid_h=4, grid_w=4, window_blocks=2, dtype=DTYPE_FP32,
                     sink_mode=SINK_AAS),
    seed=0, num_blocks=6, w_std=1.0 / np.sqrt(64.0),
    description="tiny fp32 stream: hidden 64, 1 head x 64, 4x4 grid, window 2, 6 blocks")

SUBLAYER = Workload(
    name="sublayer-14b",
    cfg=StreamConfig(num_layers=1, hidden=5120, heads=40, head_dim=128, latent_ch=5120,
                     grid_h=30, grid_w=52, window_blocks=2, timesteps=(0.5, 0.25),
                     rope_split=(22, 21, 21), sink_mode=SINK_FIXED, dtype=DTYPE_BF16),
    seed=0, num_blocks=3, w_std=0.02,
    description="one attention sublayer at 14B-DiT width, one timestep slot t=0.5")

STREAM = Workload(
    name="stream-8L",
    cfg=StreamConfig(num_layers=8, hidden=5120, heads=40, head_dim=128, latent_ch=64,
                     grid_h=30, grid_w=52, window_blocks=2, rope_split=(22, 21, 21),
                     sink_mode=SINK_AAS, dtype=DTYPE_BF16),
    seed=1, num_blocks=32, w_std=0.02,
    description="4-step timestep-forced stream, 8 sublayers, head 5120->64, 32 blocks")

SOAK = Workload(
    name="soak-2L",
    cfg=StreamConfig(num_layers=2, hidden=5120, heads=40, head_dim=128, latent_ch=64,
                     grid_h=30, grid_w=52, window_blocks=2, rope_split=(22, 21, 21),
                     sink_mode=SINK_AAS, dtype=DTYPE_BF16),
    seed=0, num_blocks=10000, w_std=0.02, fresh_step_inputs=True,
    description="10,000-block Rolling RoPE / ring soak, 2 sublayers")


def sweep_point(grid: tuple, window: int) -> Workload:
    gh, gw = grid
    return Workload(
        name=f"sweep-{gh}x{gw}-w{window}",
        cfg=StreamConfig(num_layers=1, hidden=5120, heads=40, head_dim=128, latent_ch=64,
                         grid_h=gh, grid_w=gw, window_blocks=window, rope_split=(22, 21, 21),
                         sink_mode=SINK_FIXED, dtype=DTYPE_BF16),
        seed=2, num_blocks=window + 8, w_std=0.02,
        description=f"sweep point grid {gh}x{gw}, window {window}")


SWEEP = [sweep_point(g, w) for g in ((30, 52), (45, 80)) for w in (1, 2, 4, 8)]


# ---------------------------------------------------------------------------
# Seeded draws.
# ---------------------------------------------------------------------------
def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even); returned as float32."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def _to_dtype(a: np.ndarray, dtype: int) -> np.ndarray:
    return bf16_round(a) if dtype == DTYPE_BF16 else np.ascontiguousarray(a, dtype=np.float32)


@dataclass
class Weights:
    """Weights in the [out_features, in_features] layout, already rounded to the
    config dtype (values are exactly representable in it), stored as float32."""
    w_qkv: list
    w_out: list
    w_in: Optional[np.ndarray]
    w_head: Optional[np.ndarray]
    sink: np.ndarray            # [sink_tokens, latent_ch] float32 reference sink latent
    w_ffn1: Optional[list] = None   # BLOCK_DIT: per layer [ffn_dim, hidden]
    w_ffn2: Optional[list] = None   # BLOCK_DIT: per layer [hidden, ffn_dim]
    ada: Optional[np.ndarray] = None  # BLOCK_DIT: float32 [L][num_steps + 1][6][hidden]
    w_qc: Optional[list] = None     # audio cross-attention: per layer [hidden, hidden]
    w_kvc: Optional[list] = None    # per layer [2 hidden, audio_dim] (rows 0..D-1 K, D..2D-1 V)
    w_oc: Optional[list] = None     # per layer [hidden, hidden]


def make_weights(wl: Workload) -> Weights:
    """Draw order: per layer W_qkv then W_out, then W_in, W_head, then the sink; for
    BLOCK_DIT then per layer W_ffn1, W_ffn2, then the AdaLN table, then (audio_tokens > 0)
    per layer W_qc, W_kvc (std 1/sqrt(audio_dim)), W_oc.  The AdaLN vectors
    of a (layer, timestep) are [shift1, scale1, gate1, shift2, scale2, gate2]: shifts
    and scales N(0, 0.1^2), gates N(1, 0.1^2); timestep index num_steps is t = 0."""
    c = wl.cfg
    D, C = c.hidden, c.latent_ch
    rng = np.random.default_rng(wl.seed)
    w_qkv, w_out = [], []
    for _ in range(c.num_layers):
        w_qkv.append(_to_dtype(rng.standard_normal((3 * D, D)) * wl.w_std, c.dtype))
        w_out.append(_to_dtype(rng.standard_normal((D, D)) * wl.w_std, c.dtype))
    w_in = w_head = None
    if not c.identity_in:
        w_in = _to_dtype(rng.standard_normal((D, C)) / np.sqrt(C), c.dtype)
        w_head = _to_dtype(rng.standard_normal((C, D)) * wl.head_std, c.dtype)
    sink = rng.standard_normal((c.sink_tokens, C)).astype(np.float32)
    if c.block_kind != BLOCK_DIT:
        return Weights(w_qkv, w_out, w_in, w_head, sink)
    w1, w2 = [], []
    for _ in range(c.num_layers):
        w1.append(_to_dtype(rng.standard_normal((c.ffn_dim, D)) * wl.w_std, c.dtype))
        w2.append(_to_dtype(rng.standard_normal((D, c.ffn_dim)) * wl.w_std, c.dtype))
    ada = rng.standard_normal((c.num_layers, c.num_steps + 1, 6, D)) * 0.1
    ada[:, :, 2] += 1.0
    ada[:, :, 5] += 1.0
    W = Weights(w_qkv, w_out, w_in, w_head, sink, w1, w2, ada.astype(np.float32))
    if c.audio_tokens > 0:
        W.w_qc, W.w_kvc, W.w_oc = [], [], []
        for _ in range(c.num_layers):
            W.w_qc.append(_to_dtype(rng.standard_normal((D, D)) * wl.w_std, c.dtype))
            W.w_kvc.append(_to_dtype(rng.standard_normal((2 * D, c.audio_dim)) / np.sqrt(c.audio_dim), c.dtype))
            W.w_oc.append(_to_dtype(rng.standard_normal((D, D)) * wl.w_std, c.dtype))
    return W


def block_noise(wl: Workload, b: int) -> np.ndarray:
    """Initial noise x at t_0 for block b: [block_tokens, latent_ch] float32."""
    c = wl.cfg
    return np.random.default_rng([wl.seed, b]).standard_normal(
        (c.block_tokens, c.latent_ch)).astype(np.float32)


def block_audio(wl: Workload, b: int) -> np.ndarray:
    """Audio features of block b for the cross-attention: [audio_tokens, audio_dim] float32 N(0, 1)."""
    c = wl.cfg
    return np.random.default_rng([wl.seed, b, 7]).standard_normal((c.audio_tokens, c.audio_dim)).astype(np.float32)


def step_input(wl: Workload, b: int, i: int) -> np.ndarray:
    """Fresh input of step i of block b (soak workloads)."""
    c = wl.cfg
    return np.random.default_rng([wl.seed, b, i]).standard_normal(
        (c.block_tokens, c.latent_ch)).astype(np.float32)


def random_array(seed, shape, scale=1.0) -> np.ndarray:
    """Generic seeded N(0, scale^2) float32 array for unit tests."""
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)
