"""3D rotary position embedding over (t, h, w), fp64.

The pages name RoPE and Rolling RoPE (papernotes note, 关键设计 3; admirer.cn
article, "滾動位置編碼") but give no axis split or pair layout.  Reading used
here (standard RoFormer rotary embedding, applied per axis):
  * channel pairs are interleaved, pair j = (x[2j], x[2j+1]);
  * the first p_t pairs rotate with the temporal position, the next p_h with
    the row, the last p_w with the column;
  * pair j of axis a turns by pos_a * theta^(-j / p_a);
  * rotation (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
Token order inside a block is frame-major, then row, then column.
"""
from __future__ import annotations

import numpy as np


def axis_frequencies(pairs, theta: float):
    """Per-axis angular frequencies omega_a[j] = theta^(-j/p_a), fp64."""
    out = []
    for p in pairs:
        j = np.arange(p, dtype=np.float64)
        out.append(theta ** (-j / p) if p > 0 else np.zeros(0))
    return out


def _angles(pos_t, pos_h, pos_w, pairs, theta):
    wt, wh, ww = axis_frequencies(pairs, theta)
    pos_t = np.asarray(pos_t, dtype=np.float64)[:, None]
    pos_h = np.asarray(pos_h, dtype=np.float64)[:, None]
    pos_w = np.asarray(pos_w, dtype=np.float64)[:, None]
    return np.concatenate([pos_t * wt[None, :], pos_h * wh[None, :], pos_w * ww[None, :]], axis=1)


def rope_rotate(x, pos_t, pos_h, pos_w, pairs, theta):
    """Rotate x [T, H, d] (or [T, d]) token-wise; positions are integer arrays [T]."""
    x = np.asarray(x, dtype=np.float64)
    ang = _angles(pos_t, pos_h, pos_w, pairs, theta)           # [T, P]
    if x.ndim == 3:
        ang = ang[:, None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def grid_rc(cfg):
    """Row and column of each token of one latent frame."""
    n = np.arange(cfg.frame_tokens)
    return n // cfg.grid_w, n % cfg.grid_w


def block_positions(cfg, b: int):
    """(t, h, w) integer positions of the tokens of block b: t = frames_per_block*b + f."""
    r, c = grid_rc(cfg)
    f = np.repeat(np.arange(cfg.frames_per_block), cfg.frame_tokens)
    t = cfg.frames_per_block * b + f
    return t.astype(np.int64), np.tile(r, cfg.frames_per_block), np.tile(c, cfg.frames_per_block)


def sink_temporal_position(cfg, b: int) -> int:
    """Rolling RoPE: the sink sits at (block start - offset); without rolling at -offset."""
    if cfg.rolling_rope:
        return cfg.frames_per_block * b - cfg.sink_offset_frames
    return -cfg.sink_offset_frames


def sink_positions(cfg, t_sink: int):
    r, c = grid_rc(cfg)
    nf = cfg.sink_frames
    t = np.full(cfg.frame_tokens * nf, t_sink, dtype=np.int64)
    return t, np.tile(r, nf), np.tile(c, nf)
