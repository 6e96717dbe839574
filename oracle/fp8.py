"""FP8 (e4m3) quantization, the FP8 GEMM and FP8 attention, fp64 (the operator-optimisation row).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages' largest single speed-up is operator-level optimisation (papernotes
note, inference-efficiency ablation = the paper's Table 3, last row: FP8
quantisation + FlashAttention-3 + fused kernels).  The pages give no FP8
scheme; the reading taken for the projections is per-row scaling: each row of
an operand is quantized to e4m3 with its own fp32 scale, the tensor core
multiplies the 8-bit codes exactly and accumulates, and the result is rescaled
by the row's and the column's scales:
    scale_r = amax_r / 448            (fp32; 1 for an all-zero row)
    q[r, k] = e4m3(x[r, k] / scale_r) (fp32 division, round to nearest even,
                                        saturating at +-448)
    C[m, n] = (sum_k dec(qa[m, k]) dec(qw[n, k])) * scale_a[m] * scale_w[n]

e4m3 here is the OCP 8-bit floating point format E4M3 ("FN": no infinities):
1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 is
subnormal (m/8 * 2^-6); the code with all exponent and mantissa bits set is NaN,
so the largest finite magnitude is 1.75 * 2^8 = 448.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 codes (float64; NaN for the two NaN codes)."""
    vals = np.empty(256, np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_TABLE = e4m3_decode_table()
_POS_CODES = np.arange(0x00, 0x7F)              # 0 .. 126: the non-negative finite values, increasing
_POS_VALS = _TABLE[_POS_CODES]


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round float32 values to the nearest e4m3 value, ties to the even code,
    saturating to +-448; the sign is kept, so a negative value that rounds to
    zero gives -0 (code 0x80), as IEEE rounding does.  NaN is not expected
    here.  Returns uint8 codes."""
    x = np.asarray(x, np.float32).astype(np.float64)
    mag = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS_VALS, mag, side="left")          # first value >= mag
    hi = np.clip(hi, 0, len(_POS_VALS) - 1)
    lo = np.clip(hi - 1, 0, len(_POS_VALS) - 1)
    d_hi = _POS_VALS[hi] - mag
    d_lo = mag - _POS_VALS[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (_POS_CODES[lo] % 2 == 0))
    code = np.where(pick_lo, _POS_CODES[lo], _POS_CODES[hi]).astype(np.uint8)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def bf16_round_f32(x) -> np.ndarray:
    """float32 values rounded to the nearest bfloat16 (8 significant bits, ties
    to even), returned as float32: the operand a bf16 GEMM consumes."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def project(a, w_codes, w_scales):
    """A projection on e4m3 operands: a (the bf16 operand, as float64 or
    float32 values) quantized per row, times the weight codes."""
    qa, sa = quantize_rows(bf16_round_f32(np.asarray(a, np.float64).astype(np.float32)))
    return gemm_fp8(qa, sa, w_codes, w_scales)


def quantize_rows(x):
    """Per-row e4m3 quantization: (codes uint8 [R, K], scales float32 [R])."""
    x = np.asarray(x, np.float32)
    amax = np.max(np.abs(x), axis=1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    return e4m3_encode((x / scale[:, None]).astype(np.float32)), scale


def gemm_fp8(a_codes, a_scale, w_codes, w_scale) -> np.ndarray:
    """C = (dec(A) dec(W)^T) * a_scale[:, None] * w_scale[None, :], fp64."""
    a = e4m3_decode(a_codes)
    w = e4m3_decode(w_codes)
    return (a @ w.T) * np.asarray(a_scale, np.float64)[:, None] * np.asarray(w_scale, np.float64)[None, :]


# ---- FP8 attention ---------------------------------------------------------------------
# P is formed as 2^(s - M + P_BIAS) with s the score in the log2 domain and M the
# row's largest score rounded UP to an integer, so the row's largest P lies in
# (2^(P_BIAS-1), 2^P_BIAS]: well inside e4m3's normal range, and far above its
# subnormal floor (2^-6).  Because M is an integer, scaling P by any power of two
# (another integer M) scales its e4m3 codes by the same power exactly, as long as
# the values stay normal and below 448.
P_BIAS = 5


def attention_fp8(q_codes, k_codes, v_codes, q_scale, k_scale, v_scale):
    """Softmax attention on e4m3 operands with an e4m3 probability matrix, fp64.

    The pages give no FP8 attention scheme beyond naming FP8 quantisation and
    FlashAttention-3 (papernotes note, the paper's Table 3, last row).  The
    reading taken, in FlashAttention-3's FP8 form:
      q = dec(q_codes) * q_scale[h], k and v likewise with their per-head scales;
      s[i, j] = (q_i . k_j) / sqrt(d) * log2(e)     (the log2 domain)
      M_i = ceil(max_j s[i, j])
      p[i, j] = 2^(s[i, j] - M_i + P_BIAS), rounded to float32
      O_i = sum_j dec(e4m3(p[i, j])) v_j / sum_j p[i, j]
    i.e. the product P V takes P rounded to e4m3, the normaliser takes the
    unrounded P.  Every key passed is visible (the block-causal mask is the
    choice of keys).

    q_codes: uint8 [T, H, d]; k_codes, v_codes: uint8 [N, H, d] (the visible
    keys, concatenated); scales: [H].  Returns O float64 [T, H, d]."""
    q_codes = np.asarray(q_codes, np.uint8)
    T, H, d = q_codes.shape
    out = np.empty((T, H, d), np.float64)
    for h in range(H):
        q = e4m3_decode(q_codes[:, h, :]) * float(q_scale[h])
        k = e4m3_decode(np.asarray(k_codes, np.uint8)[:, h, :]) * float(k_scale[h])
        v = e4m3_decode(np.asarray(v_codes, np.uint8)[:, h, :]) * float(v_scale[h])
        s = (q @ k.T) / np.sqrt(d) * np.log2(np.e)
        M = np.ceil(s.max(axis=1, keepdims=True))
        p = np.exp2(s - M + P_BIAS).astype(np.float32)
        pq = e4m3_decode(e4m3_encode(p))
        out[:, h, :] = (pq @ v) / p.astype(np.float64).sum(axis=1, keepdims=True)
    return out


# ---- e4m3 attention operands of the stream -------------------------------------------------
ATTN_ACT_BOUND = 1.07


def pow2_at_least(x: float) -> float:
    """The smallest power of two >= x > 0."""
    mant, ex = np.frexp(x)                  # x = mant * 2^ex, mant in [1/2, 1)
    return float(np.ldexp(1.0, int(ex) - 1 if mant == 0.5 else int(ex)))


def attn_fp8_scales(w_qkv, D: int, H: int, d: int) -> np.ndarray:
    """Per-head power-of-two scales [3, H] (q, K, V) of the stream's e4m3 attention
    operands (a reading: the pages give no FP8 scheme).  An RMS-normalised row has
    norm <= sqrt(D); its rounding to the GEMM operand grows each element by less
    than 7 % (bf16: 2^-8; per-row e4m3: 2^-4 plus the subnormal floor), so
        |value of output row j| <= 1.07 sqrt(D) ||w_j||
    by Cauchy-Schwarz, and a rotary pair (2m, 2m+1) of q or K, which RoPE mixes, is
    bounded by 1.07 sqrt(D) ||(w_2m, w_2m+1)||.  The head's scale is the smallest
    power of two with (largest bound) / scale <= 448, e4m3's largest value.
    w_qkv: the weight as the projection uses it, [3D, D] values."""
    w = np.asarray(w_qkv, np.float64)
    n2 = np.einsum("ij,ij->i", w, w)
    out = np.ones((3, H), np.float64)
    for part in range(3):
        for h in range(H):
            rows = n2[part * D + h * d: part * D + (h + 1) * d]
            m = (rows[0::2] + rows[1::2]).max() if part < 2 else rows.max()
            bound = ATTN_ACT_BOUND * np.sqrt(D) * np.sqrt(m)
            if bound > 0:
                out[part, h] = pow2_at_least(bound / E4M3_MAX)
    return out.astype(np.float32)


def quantize_heads(x, scales) -> np.ndarray:
    """e4m3 codes of x [N, H, d] over its head's scale: e4m3(float32(x) / scale[h])
    (the division by a power of two is exact)."""
    x = np.asarray(x, np.float64).astype(np.float32)
    return e4m3_encode(x / np.asarray(scales, np.float32)[None, :, None])


def dequantize_weight(codes_scales):
    """The weight a per-row e4m3 projection multiplies by: dec(codes) * row scale."""
    codes, scales = codes_scales
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[:, None]
