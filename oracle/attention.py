"""Block-causal attention with an explicit mask matrix and a naive softmax, fp64.

Definition (10100.com article, training-framework caption: causal mask over
blocks; admirer.cn article: a block only looks at earlier blocks; papernotes
note, 整体框架: 3-frame blocks, a static reference sink frame, a sliding KV
cache): a query token of block b sees
  * every sink token,
  * every token of block b' with b - window <= b' <= b (full attention inside
    the block, bidirectional),
and no other token.  Scores are q.k / sqrt(d) (scale not on the pages:
standard dot-product attention).
"""
from __future__ import annotations

import numpy as np


def block_causal_attention(q, kv_blocks: dict, sink_kv, qblock: int, window: int,
                           return_probs: bool = False):
    """q: [T, H, d]; kv_blocks: {block id: (k [Tb, H, d], v [Tb, H, d])} (roped k);
    sink_kv: (k [F, H, d], v [F, H, d]) or None.  Returns o [T, H, d]."""
    q = np.asarray(q, dtype=np.float64)
    T, H, d = q.shape
    ks, vs, key_block = [], [], []
    if sink_kv is not None:
        sk, sv = sink_kv
        ks.append(np.asarray(sk, np.float64))
        vs.append(np.asarray(sv, np.float64))
        key_block.append(np.full(sk.shape[0], -1, dtype=np.int64))
    for bid in sorted(kv_blocks):
        k, v = kv_blocks[bid]
        ks.append(np.asarray(k, np.float64))
        vs.append(np.asarray(v, np.float64))
        key_block.append(np.full(k.shape[0], bid, dtype=np.int64))
    K = np.concatenate(ks, axis=0)
    V = np.concatenate(vs, axis=0)
    kb = np.concatenate(key_block)
    # explicit [T, Nk] mask: sink always visible, window blocks and the block itself
    visible_key = (kb == -1) | ((kb >= qblock - window) & (kb <= qblock))
    mask = np.broadcast_to(visible_key[None, :], (T, K.shape[0])).copy()
    scale = 1.0 / np.sqrt(d)
    out = np.empty((T, H, d), dtype=np.float64)
    probs = []
    for h in range(H):
        s = (q[:, h, :] @ K[:, h, :].T) * scale
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ V[:, h, :]
        if return_probs:
            probs.append(p)
    if return_probs:
        return out, np.stack(probs, axis=1), mask
    return out
