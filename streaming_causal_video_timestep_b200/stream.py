"""Python binding of the streaming step: marshals torch CUDA tensors into the C ABI.

Every computation runs in libla.so's kernels; torch only provides device
memory and the CUDA stream.
"""
from __future__ import annotations

import ctypes
from ctypes import c_double, c_float, c_int32, c_int64, c_void_p

import numpy as np
import torch

from . import _lib
from ._lib import LA_EINVAL, LaConfig, LaError, LaWeights, check, load


def _dtype_code(dtype):
    return _lib.LA_BF16 if dtype in (_lib.LA_BF16, "bf16", torch.bfloat16) else _lib.LA_FP32


def torch_dtype(code):
    return torch.bfloat16 if code == _lib.LA_BF16 else torch.float32


def attn_dtype(code):
    """Element type of the attention operands (q, K, V) of a stream."""
    return torch.bfloat16 if code == _lib.LA_BF16 else torch.float32


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


def _require(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


class LaStream:
    """One avatar stream.  `cfg` is any object with the la_config fields
    (num_layers, hidden, heads, head_dim, latent_ch, grid_h, grid_w,
    frames_per_block, sink_frames, window_blocks, timesteps, rope_split or
    pairs, rope_theta, sink_mode, rolling_rope, sink_offset_frames, schedule,
    dtype, and optionally cache_mode).  `weights` holds CUDA tensors in the config dtype:
    w_qkv / w_out (lists), w_in / w_head (or None)."""

    def __init__(self, cfg, weights, stream=None):
        self.lib = load()
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        self.dtype = _dtype_code(cfg.dtype)
        self.tdtype = torch_dtype(self.dtype)
        c, self._ts = _la_config(cfg, self.dtype)
        self.cfg = cfg
        self.c = c
        self.T = cfg.frames_per_block * cfg.grid_h * cfg.grid_w
        self.F = cfg.grid_h * cfg.grid_w
        self.C, self.D = cfg.latent_ch, cfg.hidden
        self.S = c.num_steps
        # keep the weight tensors alive for the stream's lifetime (they are borrowed)
        self._weights = weights
        L = cfg.num_layers
        self._wq = (c_void_p * L)(*[w.data_ptr() for w in weights["w_qkv"]])
        self._wo = (c_void_p * L)(*[w.data_ptr() for w in weights["w_out"]])
        w = LaWeights()
        w.w_in = None if weights.get("w_in") is None else weights["w_in"].data_ptr()
        w.w_head = None if weights.get("w_head") is None else weights["w_head"].data_ptr()
        w.w_qkv = ctypes.cast(self._wq, ctypes.POINTER(c_void_p))
        w.w_out = ctypes.cast(self._wo, ctypes.POINTER(c_void_p))
        if weights.get("w_ffn1") is not None:
            # the full DiT block: FFN weights per layer and the AdaLN table (fp32 [L][S+1][6][D])
            self._w1 = (c_void_p * L)(*[t.data_ptr() for t in weights["w_ffn1"]])
            self._w2 = (c_void_p * L)(*[t.data_ptr() for t in weights["w_ffn2"]])
            S1 = len(cfg.timesteps)          # num_steps + 1 AdaLN sets
            _require(weights["ada"], torch.float32, (L, S1, 6, cfg.hidden), "ada")
            w.w_ffn1 = ctypes.cast(self._w1, ctypes.POINTER(c_void_p))
            w.w_ffn2 = ctypes.cast(self._w2, ctypes.POINTER(c_void_p))
            w.ada = weights["ada"].data_ptr()
        if weights.get("w_qc") is not None:
            # the audio cross-attention: per layer [D, D], [2D, D_a], [D, D]
            self._wqc = (c_void_p * L)(*[t.data_ptr() for t in weights["w_qc"]])
            self._wkvc = (c_void_p * L)(*[t.data_ptr() for t in weights["w_kvc"]])
            self._woc = (c_void_p * L)(*[t.data_ptr() for t in weights["w_oc"]])
            w.w_qc = ctypes.cast(self._wqc, ctypes.POINTER(c_void_p))
            w.w_kvc = ctypes.cast(self._wkvc, ctypes.POINTER(c_void_p))
            w.w_oc = ctypes.cast(self._woc, ctypes.POINTER(c_void_p))
        self.w = w
        h = c_void_p()
        code = self.lib.la_stream_create(ctypes.byref(c), ctypes.byref(w), _stream_handle(self.stream), ctypes.byref(h))
        check(code)
        self.h = h

    # -- lifecycle ----------------------------------------------------------------
    def close(self):
        if getattr(self, "h", None):
            self.lib.la_stream_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, code):
        check(code, self.h)

    # -- the four calls -------------------------------------------------------------
    def set_sink(self, latent: torch.Tensor):
        _require(latent, torch.float32, (self.F, self.C), "sink latent")
        self._check(self.lib.la_set_sink(self.h, _ptr(latent)))

    def step(self, x_new, x_out, audio=None):
        """One call of la_denoise_step (la_denoise_step_av when the stream has the audio
        cross-attention; audio: the new block's fp32 [audio_tokens, audio_dim]); returns
        the finished block id or -1."""
        if x_new is not None:
            _require(x_new, torch.float32, (self.T, self.C), "x_new")
        _require(x_out, torch.float32, (self.T, self.C), "x_out")
        fin = c_int64(-1)
        A = getattr(self.cfg, "audio_tokens", 0)
        if A > 0:
            if audio is not None:
                _require(audio, torch.float32, (A, self.cfg.audio_dim), "audio")
            self._check(self.lib.la_denoise_step_av(self.h, _ptr(x_new), _ptr(audio), _ptr(x_out),
                                                    ctypes.byref(fin)))
        else:
            self._check(self.lib.la_denoise_step(self.h, _ptr(x_new), _ptr(x_out), ctypes.byref(fin)))
        return fin.value

    def step_host(self, x_new_host, x_out_host):
        """la_denoise_step_host with (pinned) CPU tensors."""
        for t, nm in ((x_new_host, "x_new"), (x_out_host, "x_out")):
            if t is not None and (t.is_cuda or t.dtype != torch.float32 or tuple(t.shape) != (self.T, self.C)):
                raise ValueError(f"{nm} must be a CPU float32 ({self.T}, {self.C}) tensor")
        fin = c_int64(-1)
        self._check(self.lib.la_denoise_step_host(self.h, _ptr(x_new_host), _ptr(x_out_host), ctypes.byref(fin)))
        return fin.value

    def replace_sink(self, latent):
        """Slot streams (one rank of the timestep pipeline): replace the sink with frame 0
        of block 0's finished latent (device fp32 [F * sink_frames, C])."""
        _require(latent, torch.float32, (self.F * self.cfg.sink_frames, self.C), "sink latent")
        self._check(self.lib.la_replace_sink(self.h, _ptr(latent)))

    def synchronize(self):
        self._check(self.lib.la_synchronize(self.h))

    # -- debug / test ------------------------------------------------------------------
    def index_state(self) -> np.ndarray:
        n = self.lib.la_index_state_size(self.h)
        buf = (c_int32 * n)()
        self._check(self.lib.la_get_index_state(self.h, buf, n))
        return np.frombuffer(buf, dtype=np.int32).copy()

    def capture(self, enable=True):
        self._check(self.lib.la_debug_capture(self.h, 1 if enable else 0))

    def tap(self, what, layer=0, slot=0):
        T, C, D, F = self.T, self.C, self.D, self.F
        H, d, E = self.cfg.heads, self.cfg.head_dim, self.cfg.window_blocks + 1
        dt = self.tdtype
        shapes = {
            "x_in": ((T, C), torch.float32), "x_out": ((T, C), torch.float32), "v": ((T, C), torch.float32),
            "h": ((T, D), torch.float32), "q": ((H, T, d), dt), "o": ((T, D), dt),
            "ring_k": ((E, H, T, d), dt), "ring_v": ((E, H, T, d), dt), "sink_k": ((H, F, d), dt),
            "sink_v": ((H, F, d), dt), "sink_k_rope": ((H, F, d), dt), "sink_h": ((F, D), torch.float32),
            "hop": ((T, D), dt), "sink_hop": ((F, D), dt),
            "sink_v8": ((H, F, d), torch.uint8), "attn_scales": ((3, H), torch.float32),
            "h_mid": ((T, D), torch.float32), "ffn_u": ((T, max(1, getattr(self.cfg, "ffn_dim", 0))), dt),
            "h_cross": ((T, D), torch.float32), "xo": ((T, D), torch.float32), "xq": ((H, T, d), dt),
            "xk": ((H, max(1, getattr(self.cfg, "audio_tokens", 0)), d), dt),
            "xv": ((H, max(1, getattr(self.cfg, "audio_tokens", 0)), d), dt),
        }
        shape, tdt = shapes[what]
        if what in ("xq", "xk", "xv"):
            tdt = attn_dtype(self.dtype)
        elif what in ("q", "ring_k", "ring_v", "sink_k_rope") and getattr(self.cfg, "attn_fp8", 0):
            tdt = torch.uint8          # e4m3 codes
        elif what in ("q", "ring_k", "ring_v", "sink_v", "sink_k_rope"):
            tdt = attn_dtype(self.dtype)
        elif what in ("o", "sink_k"):
            tdt = torch.float32
        out = torch.empty(shape, dtype=tdt, device="cuda")
        self._check(self.lib.la_debug_tap(self.h, _lib.TAP[what], layer, slot, _ptr(out),
                                          out.numel() * out.element_size()))
        return out

    def set_slot_input(self, slot, x):
        _require(x, torch.float32, (self.T, self.C), "slot input")
        self._check(self.lib.la_debug_set_slot_input(self.h, slot, _ptr(x)))

    def profile(self, enable=True):
        self._check(self.lib.la_profile_enable(self.h, 1 if enable else 0))

    def profile_read(self, kind):
        n, ms = c_int64(0), c_double(0.0)
        self._check(self.lib.la_profile_read(self.h, _lib.KIND[kind], ctypes.byref(n), ctypes.byref(ms)))
        return n.value, ms.value

    def launch_count(self):
        return self.lib.la_launch_count(self.h)


def _la_config(cfg, dtype_code):
    """The C configuration of cfg, and the timestep array it points into (keep it alive)."""
    ts = [float(t) for t in cfg.timesteps]
    ts_arr = (c_float * len(ts))(*ts)
    pairs = getattr(cfg, "pairs", None) or cfg.rope_split
    c = LaConfig()
    c.num_layers, c.hidden, c.heads, c.head_dim = cfg.num_layers, cfg.hidden, cfg.heads, cfg.head_dim
    c.latent_ch, c.grid_h, c.grid_w = cfg.latent_ch, cfg.grid_h, cfg.grid_w
    c.frames_per_block, c.sink_frames, c.window_blocks = cfg.frames_per_block, cfg.sink_frames, cfg.window_blocks
    c.num_steps = len(ts) - 1
    c.timesteps = ctypes.cast(ts_arr, ctypes.POINTER(c_float))
    c.rope_split = (c_int32 * 3)(*pairs)
    c.rope_theta = float(cfg.rope_theta)
    c.sink_mode, c.rolling_rope, c.sink_offset_frames = cfg.sink_mode, cfg.rolling_rope, cfg.sink_offset_frames
    c.schedule, c.dtype = cfg.schedule, dtype_code
    c.cache_mode = getattr(cfg, "cache_mode", 0)
    c.proj_fp8 = getattr(cfg, "proj_fp8", 0)
    c.attn_fp8 = getattr(cfg, "attn_fp8", 0)
    c.cache_step = getattr(cfg, "cache_step", 0)
    c.block_kind = getattr(cfg, "block_kind", 0)
    c.ffn_dim = getattr(cfg, "ffn_dim", 0)
    c.audio_tokens = getattr(cfg, "audio_tokens", 0)
    c.audio_dim = getattr(cfg, "audio_dim", 0)
    c.slot_index = getattr(cfg, "slot_index", 0)
    return c, ts_arr


def sched_trace(cfg, has_new):
    """The tick scheduler alone, on the host (la_sched_trace; no GPU): the index
    state after each of len(has_new) calls (has_new[k]: call k brings a new
    block), int32 [calls, la_sched_state_size]."""
    lib = load()
    c, _keep = _la_config(cfg, _dtype_code(cfg.dtype))
    size = lib.la_sched_state_size(ctypes.byref(c))
    if size < 0:
        raise LaError(LA_EINVAL, "bad scheduling configuration")
    n = len(has_new)
    flags = (ctypes.c_uint8 * max(n, 1))(*[1 if x else 0 for x in has_new])
    out = np.zeros((n, size), np.int32)
    check(lib.la_sched_trace(ctypes.byref(c), n, flags, out.ctypes.data_as(ctypes.POINTER(c_int32)), out.size))
    return out


# ---- op-level wrappers -------------------------------------------------------------------
def op_gemm(A, W, epilogue="store", out=None, h32=None, dt=None, rows_per_group=0, stream=None):
    lib = load()
    dtype = _dtype_code(A.dtype)
    M, K = A.shape
    N = W.shape[0]
    epi = dict(store=_lib.LA_EPI_STORE, resid=_lib.LA_EPI_RESID, set32=_lib.LA_EPI_SET32,
               euler=_lib.LA_EPI_EULER, store32=_lib.LA_EPI_STORE32)[epilogue]
    dtp = None
    if dt is not None:
        dtp = (c_float * len(dt))(*[float(x) for x in dt])
    code = lib.la_op_gemm(dtype, epi, _ptr(A), _ptr(W), _ptr(out), _ptr(h32), M, N, K, dtp, rows_per_group,
                          _stream_handle(stream))
    check(code)


def op_attention(q, ks, vs, out, out32=None, q_scaled=False, stream=None):
    """q [H, Tq, d] bf16 (tcgen05) or fp32 (SIMT); ks / vs lists of [H, len, d];
    out [Tq, H*d] in the input type; out32 optional fp32 copy; q_scaled: q is
    already multiplied by log2(e)/sqrt(d) (bf16 only)."""
    lib = load()
    dtype = _dtype_code(q.dtype)
    H, Tq, d = q.shape
    n = len(ks)
    kp = (c_void_p * n)(*[k.data_ptr() for k in ks])
    vp = (c_void_p * n)(*[v.data_ptr() for v in vs])
    ln = (c_int64 * n)(*[k.shape[1] for k in ks])
    code = lib.la_op_attention(dtype, _ptr(q), Tq, H, d, n, kp, vp, ln, _ptr(out), _ptr(out32),
                               1 if q_scaled else 0, _stream_handle(stream))
    check(code)


def op_euler(x, v, dt, rows_per_group, stream=None):
    lib = load()
    rows, C = x.shape
    dtp = (c_float * len(dt))(*[float(t) for t in dt])
    check(lib.la_op_euler(_ptr(x), _ptr(v), rows, C, dtp, rows_per_group, _stream_handle(stream)))


def op_quantize_e4m3(x, codes, scales, stream=None):
    """Per-row e4m3 quantization: x [rows, cols] bf16 or fp32 CUDA tensor ->
    codes uint8 [rows, cols], scales fp32 [rows] (amax / 448)."""
    lib = load()
    rows, cols = x.shape
    check(lib.la_op_quantize_e4m3(_dtype_code(x.dtype), _ptr(x), rows, cols, _ptr(codes), _ptr(scales),
                                  _stream_handle(stream)))


def op_gemm_fp8(a_codes, a_scales, w_codes, w_scales, out, stream=None):
    """out [M, N] (bf16 or fp32) = (A W^T) * a_scales[:, None] * w_scales[None, :] from
    uint8 e4m3 codes A [M, K], W [N, K] on the tensor cores."""
    lib = load()
    M, K = a_codes.shape
    N = w_codes.shape[0]
    check(lib.la_op_gemm_fp8(_ptr(a_codes), _ptr(a_scales), _ptr(w_codes), _ptr(w_scales), _ptr(out),
                             _dtype_code(out.dtype), M, N, K, _stream_handle(stream)))


def op_attention_fp8(q_codes, ks, vs, q_scale, k_scale, v_scale, out, out32=None, stream=None):
    """FP8 attention: q_codes [H, Tq, 128] uint8 e4m3; ks / vs lists of uint8 [H, len, 128];
    q_scale / k_scale / v_scale fp32 [H] CUDA tensors; out bf16 [Tq, H*128], out32 optional
    fp32 copy."""
    lib = load()
    H, Tq, d = q_codes.shape
    n = len(ks)
    kp = (c_void_p * n)(*[k.data_ptr() for k in ks])
    vp = (c_void_p * n)(*[v.data_ptr() for v in vs])
    ln = (c_int64 * n)(*[k.shape[1] for k in ks])
    check(lib.la_op_attention_fp8(_ptr(q_codes), Tq, H, d, n, kp, vp, ln, _ptr(q_scale), _ptr(k_scale),
                                  _ptr(v_scale), _ptr(out), _ptr(out32), _stream_handle(stream)))
