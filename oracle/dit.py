"""The full synthetic DiT block (AdaLN-modulated attention and FFN sub-blocks), fp64.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages give the model's base (a 14B DiT, WanS2V, with timestep
conditioning; papernotes note, 整体框架 and 损失函数) but no layer internals.
Reading, after the Wan-style DiT block the model is built on: each layer is
    m1 = n(h) * (1 + scale1) + shift1                  (AdaLN)
    h  = h + gate1 * Attn(m1)                          (the attention sublayer's
                                                        QKV / RoPE / cache / attention
                                                        / output projection)
    m2 = n(h) * (1 + scale2) + shift2
    h  = h + gate2 * (gelu(m2 W1^T) W2^T)              (FFN, tanh GELU)
with n the per-token RMS norm (oracle/norm.py) and (shift1, scale1, gate1,
shift2, scale2, gate2) the AdaLN vectors of the layer at the step's timestep:
the timestep embedding and its projection are fixed for the 4 distilled
timesteps, so the library takes the vectors themselves as weights, one set per
(layer, timestep) plus one for t = 0 (the clean sink frame and the clean-cache
refresh).

Audio cross-attention (the model is audio-driven; papernotes note, 整体框架;
reading: Wan's cross-attention sub-block, between the attention and the FFN):
    h = h + (softmax(q k^T / sqrt(d)) v) W_oc^T,  q = n(h) W_qc^T,
    [k | v] = audio_b W_kvc^T
over all audio tokens of the block (no RoPE, no mask; heads as in the
self-attention).  The sink frame has no audio: its pass skips the sub-block.
"""
from __future__ import annotations

import numpy as np

from .norm import rms_norm

GELU_C = np.sqrt(2.0 / np.pi)


def gelu_tanh(u):
    """GELU with the tanh approximation: u/2 (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    u = np.asarray(u, np.float64)
    return 0.5 * u * (1.0 + np.tanh(GELU_C * (u + 0.044715 * u ** 3)))


def modulate(h, shift, scale):
    """AdaLN: n(h) * (1 + scale) + shift, per token; shift / scale [D]."""
    return rms_norm(h) * (1.0 + np.asarray(scale, np.float64)) + np.asarray(shift, np.float64)


def ffn(m, w1, w2):
    """gelu(m W1^T) W2^T; w1 [F, D], w2 [D, F]."""
    return gelu_tanh(np.asarray(m, np.float64) @ np.asarray(w1, np.float64).T) @ np.asarray(w2, np.float64).T


def cross_attention(h, audio, w_qc, w_kvc, w_oc, heads, head_dim):
    """The audio cross-attention sub-block's contribution (to be added to h):
    softmax(q k^T / sqrt(d)) v W_oc^T with q = n(h) W_qc^T and [k | v] = audio W_kvc^T."""
    from .attention import block_causal_attention
    h = np.asarray(h, np.float64)
    T, D = h.shape
    q = (rms_norm(h) @ np.asarray(w_qc, np.float64).T).reshape(T, heads, head_dim)
    kv = np.asarray(audio, np.float64) @ np.asarray(w_kvc, np.float64).T
    A = kv.shape[0]
    k = kv[:, :D].reshape(A, heads, head_dim)
    v = kv[:, D:].reshape(A, heads, head_dim)
    o = block_causal_attention(q, {0: (k, v)}, None, qblock=0, window=0)
    return o.reshape(T, D) @ np.asarray(w_oc, np.float64).T
