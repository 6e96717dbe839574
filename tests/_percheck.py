"""Per-op teacher-forced parity of one captured (block, step) of a stream.

Each kernel of the step is checked against the oracle's definition applied to
the GPU's own inputs to that kernel (the tolerance is stated for bf16 inputs
with fp32 accumulation): the in-projection from the captured latent, QKV +
Rolling RoPE + ring append from the captured residual rounded to the GEMM
operand type, the sink re-rope from the stored un-roped sink K, attention from
the captured q and the ring / sink tensors, the output projection from the
attention output as the next GEMM consumes it, and the head + Euler update.
`rows` restricts the row-wise checks to a sample of query rows (full-size
streams); attention keys are always complete.
"""
import numpy as np

import math

from oracle import RMS_EPS, block_causal_attention, euler_step, rms_norm, rope_rotate
from oracle.dit import gelu_tanh, modulate
from oracle.fp8 import (attention_fp8, attn_fp8_scales, dequantize_weight, project, quantize_heads,
                        quantize_rows)
from oracle.rope import block_positions, sink_positions
from workloads import CACHE_FIXED_STEP, DTYPE_BF16, bf16_round

from _helpers import assert_close, to_np


def _operand(a, cfg):
    """The value a GEMM consumes: bf16-rounded in bf16 streams, fp32 in fp32 streams."""
    a = np.asarray(a, np.float32)
    return bf16_round(a).astype(np.float64) if cfg.dtype == DTYPE_BF16 else a.astype(np.float64)


def _normed_operand(h, cfg):
    """The per-token RMS-normalised residual as the next GEMM consumes it."""
    return _operand(rms_norm(np.asarray(h, np.float64)).astype(np.float32), cfg)


def _dit(cfg):
    return getattr(cfg, "block_kind", 0) == 1


def _folded(cfg, W):
    """Whether the stream folds the RMS norm into its GEMMs (bf16 attention
    sublayers with an in-projection and a head): the QKV and head GEMMs then
    consume the residual itself rounded to bf16 (with e4m3 projections, quantized
    per row from it), and scale each product row by the row's 1 / rms, taken from
    the fp32 residual."""
    return (cfg.dtype == DTYPE_BF16 and not _dit(cfg)
            and W.w_in is not None and W.w_head is not None)


def _inv_rms(h):
    h = np.asarray(h, np.float64)
    return 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + RMS_EPS)


def _attn_operand(h, cfg, W, l, t_idx):
    """The QKV projection's operand: the normalised residual, AdaLN-modulated in the DiT block."""
    if not _dit(cfg):
        return _normed_operand(h, cfg)
    a = np.asarray(W.ada, np.float64)[l, t_idx]
    return _operand(modulate(np.asarray(h, np.float64), a[0], a[1]).astype(np.float32), cfg)


_W8 = {}


def _proj(a, w, cfg):
    """A QKV / output projection of the operand a (as the GEMM consumes it): bf16
    or fp32 GEMM, or with e4m3 projections (cfg.proj_fp8) the quantized operand
    times the per-row-quantized weights (oracle/fp8.py)."""
    if not getattr(cfg, "proj_fp8", 0):
        return a @ np.asarray(w, np.float64).T
    hit = _W8.get(id(w))
    if hit is None or hit[0] is not w:
        hit = (w, quantize_rows(np.asarray(w, np.float32)))
        _W8[id(w)] = hit
    return project(a, *hit[1])


def _qkv_weight_used(w, cfg):
    """The QKV weight as the projection multiplies it (dequantized e4m3 with proj_fp8)."""
    if not getattr(cfg, "proj_fp8", 0):
        return np.asarray(w, np.float64)
    _proj(np.zeros((1, w.shape[1])), w, cfg)            # fills the quantized-weight cache
    return dequantize_weight(_W8[id(w)][1])


_SC = {}


def attn_scales(s, cfg, W, l):
    """The GPU's per-head e4m3 scales of layer l, checked equal to the oracle's rule."""
    sc = to_np(s.tap("attn_scales", l)).astype(np.float32)
    key = (id(W.w_qkv[l]), getattr(cfg, "proj_fp8", 0))
    if key not in _SC:
        _SC[key] = attn_fp8_scales(_qkv_weight_used(W.w_qkv[l], cfg), cfg.hidden, cfg.heads, cfg.head_dim)
    np.testing.assert_array_equal(sc, _SC[key])
    return sc


def check_codes(codes, x, scales, what):
    """e4m3 codes of the GPU against the oracle's quantization of its own value x
    [N, H, d] (quantize_heads).  The GPU quantizes its fp32 result, which differs from
    the oracle's by the GEMM's accumulation rounding, so a value at a rounding tie may
    take the neighbouring code: every difference must be to an adjacent code of the
    same sign, and at most 1 % of the codes may differ.  Returns the fraction."""
    want = quantize_heads(x, scales)
    codes = np.asarray(codes, np.uint8)
    diff = codes != want
    frac = float(diff.mean())
    if diff.any():
        g, w_ = codes[diff].astype(np.int32), want[diff].astype(np.int32)
        mag_g, mag_w = g & 0x7F, w_ & 0x7F
        same_sign = ((g & 0x80) == (w_ & 0x80)) | ((mag_g == 0) & (mag_w == 0)) | (np.maximum(mag_g, mag_w) <= 1)
        adjacent = np.abs(mag_g - mag_w) <= 1
        assert np.all(same_sign & adjacent), f"{what}: non-adjacent e4m3 code"
    assert frac <= 1e-2, f"{what}: {frac:.2e} of the codes differ"
    return frac


def _window_rings(s, cfg, l, i, ring_k, ring_v):
    """The rings step i reads its prior blocks from: its own, or with the fixed-noise
    cache step cache_step's ([E, T, H, d] each)."""
    if getattr(cfg, "cache_mode", 0) != CACHE_FIXED_STEP or cfg.cache_step == i:
        return ring_k, ring_v
    j = cfg.cache_step
    return (to_np(s.tap("ring_k", l, j)).transpose(0, 2, 1, 3), to_np(s.tap("ring_v", l, j)).transpose(0, 2, 1, 3))


def check_sink(s, cfg, W, latent, rows=None, tag=""):
    """Per-op check of the last sink pass: in-projection of the sink latent and,
    per layer, the stored un-roped K (fp32) and V from the captured sink residual."""
    dt = cfg.dtype
    F, D, H, d = cfg.sink_tokens, cfg.hidden, cfg.heads, cfg.head_dim
    R = np.arange(F) if rows is None else np.asarray(rows)
    h0 = to_np(s.tap("sink_h", 0))
    lat = np.asarray(latent, np.float64)
    want = lat[R] if W.w_in is None else _operand(lat[R], cfg) @ np.asarray(W.w_in, np.float64).T
    assert_close(h0[R], want, dt, f"{tag} sink in-proj")
    for l in range(cfg.num_layers):
        hs = to_np(s.tap("sink_h", l))
        op = _attn_operand(hs[R], cfg, W, l, cfg.num_steps)
        if getattr(cfg, "proj_fp8", 0) or getattr(cfg, "attn_fp8", 0):
            # e4m3 operands downstream: the normalisation on its own, then the projection
            # from the operand the GPU consumed (a one-ulp difference there can move
            # a code, or a row's scale, by a whole e4m3 step)
            op_gpu = to_np(s.tap("sink_hop", l))[R].astype(np.float64)
            assert_close(op_gpu, op, dt, f"{tag} sink norm operand l{l}")
            op = op_gpu
        qkv = _proj(op, W.w_qkv[l], cfg)
        k = qkv[:, D:2 * D].reshape(len(R), H, d)
        v = qkv[:, 2 * D:].reshape(len(R), H, d)
        assert_close(to_np(s.tap("sink_k", l)).transpose(1, 0, 2)[R], k, dt, f"{tag} sink K l{l}")
        assert_close(to_np(s.tap("sink_v", l)).transpose(1, 0, 2)[R], v, dt, f"{tag} sink V l{l}")
        if getattr(cfg, "attn_fp8", 0):
            sc = attn_scales(s, cfg, W, l)
            check_codes(to_np(s.tap("sink_v8", l)).transpose(1, 0, 2)[R], v, sc[2], f"{tag} sink V codes l{l}")


def sink_snapshot(s, cfg):
    """The sink K (un-roped) and V of every layer as they are now: take it before
    a call whose per-op check follows (the AAS replacement at the end of the
    call that finishes block 0 changes them)."""
    snap = ([to_np(s.tap("sink_k", l)).transpose(1, 0, 2) for l in range(cfg.num_layers)],
            [to_np(s.tap("sink_v", l)).transpose(1, 0, 2) for l in range(cfg.num_layers)])
    if getattr(cfg, "attn_fp8", 0):
        snap += ([to_np(s.tap("sink_v8", l)).transpose(1, 0, 2) for l in range(cfg.num_layers)],)
    return snap


def check_step(s, cfg, W, b, i, rows=None, tag="", report=None, sink=None, audio=None):
    """sink: sink_snapshot() taken before the call (default: the current sink); audio:
    block b's audio features (streams with the audio cross-attention)."""
    dt = cfg.dtype
    T, D, H, d, E, L = cfg.block_tokens, cfg.hidden, cfg.heads, cfg.head_dim, cfg.ring_entries, cfg.num_layers
    R = np.arange(T) if rows is None else np.asarray(rows)
    f64 = lambda a: None if a is None else np.asarray(a, np.float64)
    w_in, w_head = f64(W.w_in), f64(W.w_head)
    pt, ph, pw = block_positions(cfg, b)
    st = sink_positions(cfg, (cfg.frames_per_block * b - cfg.sink_offset_frames) if cfg.rolling_rope
                        else -cfg.sink_offset_frames)
    errs = {}

    def chk(got, want, what):
        e = assert_close(got, want, dt, f"{tag} {what} b{b} s{i}")
        errs[what] = max(errs.get(what, (0, 0)), e)

    x_in = to_np(s.tap("x_in", 0, i)).astype(np.float64)
    h_in = to_np(s.tap("h", -1, i))
    want = x_in[R] if w_in is None else _operand(x_in[R], cfg) @ w_in.T
    chk(h_in[R], want, "in-proj h")
    h_prev = h_in
    fold = _folded(cfg, W)
    for l in range(L):
        # folded norm: n(h) W^T taken as diag(1 / rms(h)) (bf16(h) W^T)
        op = _operand(h_prev[R], cfg) if fold else _attn_operand(h_prev[R], cfg, W, l, i)
        rs = _inv_rms(h_prev[R]) if fold else 1.0
        if getattr(cfg, "proj_fp8", 0) or getattr(cfg, "attn_fp8", 0):
            # e4m3 operands downstream: check the normalisation on its own, then go on
            # from the operand the GPU consumed (a one-ulp bf16 difference there moves
            # a product by more than the rounding an e4m3 code check can absorb)
            op_gpu = to_np(s.tap("hop", l, i))[R].astype(np.float64)
            chk(op_gpu, op, f"norm operand l{l}")
            op = op_gpu
        qkv = _proj(op, W.w_qkv[l], cfg) * rs
        q = qkv[:, :D].reshape(len(R), H, d)
        k = qkv[:, D:2 * D].reshape(len(R), H, d)
        v = qkv[:, 2 * D:].reshape(len(R), H, d)
        qr = rope_rotate(q, pt[R], ph[R], pw[R], cfg.pairs, cfg.rope_theta)
        kr = rope_rotate(k, pt[R], ph[R], pw[R], cfg.pairs, cfg.rope_theta)
        if getattr(cfg, "attn_fp8", 0):
            _check_attn_fp8(s, cfg, W, b, i, l, R, qr, kr, v, sink, st, chk, errs, tag)
            o_gpu = to_np(s.tap("o", l, i))
            h_next = to_np(s.tap("h", l, i))
            want = h_prev[R].astype(np.float64) + _proj(_operand(o_gpu[R], cfg), W.w_out[l], cfg)
            chk(h_next[R], want, f"h l{l}")
            h_prev = h_next
            continue
        q_gpu = to_np(s.tap("q", l, i)).transpose(1, 0, 2)           # [T, H, d]
        if dt == DTYPE_BF16:
            # bf16 streams store q pre-multiplied by the softmax scale log2(e)/sqrt(d)
            qscale = float(np.float32(math.log2(math.e) / math.sqrt(d)))
            qr = qr * qscale
            q_att = q_gpu / qscale
        else:
            q_att = q_gpu
        ring_k = to_np(s.tap("ring_k", l, i)).transpose(0, 2, 1, 3)  # [E, T, H, d]
        ring_v = to_np(s.tap("ring_v", l, i)).transpose(0, 2, 1, 3)
        win_k, win_v = _window_rings(s, cfg, l, i, ring_k, ring_v)
        e = b % E
        chk(q_gpu[R], qr, f"q l{l}")
        chk(ring_k[e][R], kr, f"ring K l{l}")
        chk(ring_v[e][R], v, f"ring V l{l}")
        # sink re-rope for this block from the stored fp32 un-roped sink K
        sk_raw = sink[0][l] if sink is not None else to_np(s.tap("sink_k", l)).transpose(1, 0, 2)
        sk_rope = to_np(s.tap("sink_k_rope", l, i)).transpose(1, 0, 2)
        chk(sk_rope, rope_rotate(sk_raw, *st, cfg.pairs, cfg.rope_theta), f"sink K rope l{l}")
        sv = sink[1][l] if sink is not None else to_np(s.tap("sink_v", l)).transpose(1, 0, 2)
        # attention from the GPU's own q and cache contents
        blocks = {bb: (win_k[bb % E], win_v[bb % E]) for bb in range(max(0, b - cfg.window_blocks), b)}
        blocks[b] = (ring_k[e], ring_v[e])
        o_want = block_causal_attention(q_att[R], blocks, (sk_rope, sv), qblock=b, window=cfg.window_blocks)
        o_gpu = to_np(s.tap("o", l, i))
        chk(o_gpu[R], o_want.reshape(len(R), D), f"attn O l{l}")
        # output projection + residual from the attention output as the GEMM consumes it
        h_next = to_np(s.tap("h", l, i))
        if _dit(cfg):
            _check_ffn(s, cfg, W, l, i, R, h_prev, o_gpu, h_next, chk, audio)
            h_prev = h_next
            continue
        want = h_prev[R].astype(np.float64) + _proj(_operand(o_gpu[R], cfg), W.w_out[l], cfg)
        chk(h_next[R], want, f"h l{l}")
        h_prev = h_next
    if w_head is None:
        vel = rms_norm(h_prev[R].astype(np.float64))
    elif fold:
        vel = (_operand(h_prev[R], cfg) @ w_head.T) * _inv_rms(h_prev[R])
    else:
        vel = _normed_operand(h_prev[R], cfg) @ w_head.T
    chk(to_np(s.tap("v", 0, i))[R], vel, "velocity")
    x_want = euler_step(x_in[R], vel, cfg.timesteps[i], cfg.timesteps[i + 1])
    chk(to_np(s.tap("x_out", 0, i))[R], x_want, "x")
    if report is not None:
        for k_, v_ in errs.items():
            report[k_] = max(report.get(k_, (0, 0)), v_)
    return errs


def _check_attn_fp8(s, cfg, W, b, i, l, R, qr, kr, v, sink, st, chk, errs, tag):
    """e4m3 attention of one layer: scales, the codes of q / the ring entry / the
    re-roped sink K against the oracle's values, then the attention from the GPU's
    own codes (oracle.fp8.attention_fp8)."""
    E, D = cfg.ring_entries, cfg.hidden
    sc = attn_scales(s, cfg, W, l)
    q8 = to_np(s.tap("q", l, i)).transpose(1, 0, 2)                  # [T, H, d] codes
    rk8 = to_np(s.tap("ring_k", l, i)).transpose(0, 2, 1, 3)         # [E, T, H, d]
    rv8 = to_np(s.tap("ring_v", l, i)).transpose(0, 2, 1, 3)
    e = b % E
    fr = {}
    fr["q codes"] = check_codes(q8[R], qr, sc[0], f"{tag} q codes l{l} b{b} s{i}")
    fr["ring K codes"] = check_codes(rk8[e][R], kr, sc[1], f"{tag} ring K codes l{l} b{b} s{i}")
    fr["ring V codes"] = check_codes(rv8[e][R], v, sc[2], f"{tag} ring V codes l{l} b{b} s{i}")
    sk_raw = sink[0][l] if sink is not None else to_np(s.tap("sink_k", l)).transpose(1, 0, 2)
    sk8 = to_np(s.tap("sink_k_rope", l, i)).transpose(1, 0, 2)
    fr["sink K codes"] = check_codes(sk8, rope_rotate(sk_raw, *st, cfg.pairs, cfg.rope_theta), sc[1],
                                     f"{tag} sink K codes l{l} b{b} s{i}")
    sv8 = sink[2][l] if sink is not None and len(sink) > 2 else to_np(s.tap("sink_v8", l)).transpose(1, 0, 2)
    wk8, wv8 = _window_rings(s, cfg, l, i, rk8, rv8)
    order = range(max(0, b - cfg.window_blocks), b)
    keys = np.concatenate([sk8] + [wk8[bb % E] for bb in order] + [rk8[e]])
    vals = np.concatenate([sv8] + [wv8[bb % E] for bb in order] + [rv8[e]])
    o_want = attention_fp8(q8[R], keys, vals, sc[0], sc[1], sc[2])
    chk(to_np(s.tap("o", l, i))[R], o_want.reshape(len(R), D), f"attn O (e4m3) l{l}")
    for k_, f_ in fr.items():
        errs[k_] = max(errs.get(k_, (0, 0)), (f_, 0.0))


def _check_ffn(s, cfg, W, l, i, R, h_prev, o_gpu, h_next, chk, audio=None):
    """The DiT block after attention: the gated output projection (h_mid), the audio
    cross-attention (when the stream has audio), the AdaLN-modulated FFN operand and
    its GELU output (u), and the gated FFN residual, each from the GPU's own inputs."""
    a = np.asarray(W.ada, np.float64)[l, i]
    h_mid = to_np(s.tap("h_mid", l, i))
    want = h_prev[R].astype(np.float64) + a[2] * _proj(_operand(o_gpu[R], cfg), W.w_out[l], cfg)
    chk(h_mid[R], want, f"h mid l{l}")
    if getattr(cfg, "audio_tokens", 0) > 0:
        h_mid = _check_cross(s, cfg, W, l, i, R, h_mid, audio, chk)
    m2 = _operand(modulate(h_mid[R].astype(np.float64), a[3], a[4]).astype(np.float32), cfg)
    u_gpu = to_np(s.tap("ffn_u", l, i))
    chk(u_gpu[R], gelu_tanh(m2 @ np.asarray(W.w_ffn1[l], np.float64).T), f"ffn gelu l{l}")
    want = h_mid[R].astype(np.float64) + a[5] * (_operand(u_gpu[R], cfg) @ np.asarray(W.w_ffn2[l], np.float64).T)
    chk(h_next[R], want, f"h l{l}")


def _check_cross(s, cfg, W, l, i, R, h_mid, audio, chk):
    """The audio cross-attention sub-block from the GPU's inputs: its q from the
    residual, the block's audio K / V, the attention from the GPU's q / K / V, and
    the residual after the output projection.  Returns the GPU's residual after it."""
    D, H, d = cfg.hidden, cfg.heads, cfg.head_dim
    q_want = (_normed_operand(h_mid[R], cfg) @ np.asarray(W.w_qc[l], np.float64).T).reshape(len(R), H, d)
    xq = to_np(s.tap("xq", l, i)).transpose(1, 0, 2)                 # [T, H, d]
    qs = float(np.float32(math.log2(math.e) / math.sqrt(d))) if cfg.dtype == DTYPE_BF16 else 1.0
    chk(xq[R] / qs, q_want, f"cross q l{l}")
    kv = _operand(np.asarray(audio, np.float32), cfg) @ np.asarray(W.w_kvc[l], np.float64).T
    A = kv.shape[0]
    xk = to_np(s.tap("xk", l, i)).transpose(1, 0, 2)                 # [A, H, d]
    xv = to_np(s.tap("xv", l, i)).transpose(1, 0, 2)
    chk(xk, kv[:, :D].reshape(A, H, d), f"cross K l{l}")
    chk(xv, kv[:, D:].reshape(A, H, d), f"cross V l{l}")
    o_want = block_causal_attention(xq[R] / qs, {0: (xk, xv)}, None, qblock=0, window=0)
    xo = to_np(s.tap("xo", l, i))
    chk(xo[R], o_want.reshape(len(R), D), f"cross O l{l}")
    h_x = to_np(s.tap("h_cross", l, i))
    want = h_mid[R].astype(np.float64) + _operand(xo[R], cfg) @ np.asarray(W.w_oc[l], np.float64).T
    chk(h_x[R], want, f"h cross l{l}")
    return h_x
