"""Pins of the oracle's e4m3 quantization and FP8 GEMM (CPU only).

The decode table and the rounding are checked against torch's float8_e4m3fn
(a library implementation of the same OCP format) and against values fixed by
the format's definition; the GEMM against a product of torch-decoded operands.
"""
import numpy as np
import pytest
import torch

from oracle.fp8 import E4M3_MAX, bf16_round_f32, e4m3_decode, e4m3_decode_table, e4m3_encode, gemm_fp8, quantize_rows


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn).float().numpy()


def test_decode_table_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_decode_table()
    ref = _torch_decode(codes).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])


def test_values_fixed_by_the_format():
    t = e4m3_decode_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0            # largest finite: 1.75 * 2^8
    assert t[0x01] == 2.0 ** -9                               # smallest subnormal: 1/8 * 2^-6
    assert t[0x08] == 2.0 ** -6                               # smallest normal
    assert t[0x38] == 1.0                                     # exponent field 7 = bias
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.count_nonzero(np.isnan(t)) == 2


def test_encode_matches_torch_rounding_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(200000) * 30, rng.uniform(-463, 463, 100000),
                        rng.standard_normal(50000) * 1e-2, rng.standard_normal(50000) * 1e-3]).astype(np.float32)
    x = np.concatenate([x, np.float32([-1e-5, 1e-5, -0.0, 0.0, -2.0 ** -10])])   # signed zeros
    ours = e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_ties_go_to_the_even_code_and_large_values_saturate():
    half_sub = np.float32(2.0 ** -10)           # halfway between 0 and the smallest subnormal
    assert e4m3_encode([half_sub])[0] == 0x00
    assert e4m3_encode([np.float32(3 * 2.0 ** -10)])[0] == 0x02      # between codes 1 and 2 -> 2
    assert e4m3_encode([np.float32(1.0625)])[0] == 0x38               # between 1.0 (0x38) and 1.125 (0x39)
    assert e4m3_encode([np.float32(1.1875)])[0] == 0x3A               # between 0x39 and 0x3A -> 0x3A
    assert list(e4m3_encode([1000.0, -1e30, 448.0, 463.9])) == [0x7E, 0xFE, 0x7E, 0x7E]


def test_quantize_rows_maps_each_row_max_to_448_and_bounds_the_error():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 1000)) * rng.uniform(0.01, 100, (64, 1))).astype(np.float32)
    x[5] = 0.0
    q, s = quantize_rows(x)
    assert s[5] == 1.0 and not q[5].any()
    deq = e4m3_decode(q) * s[:, None]
    rows = [r for r in range(64) if r != 5]
    amax_idx = np.argmax(np.abs(x), axis=1)
    for r in rows:
        assert abs(e4m3_decode(q[r, amax_idx[r]])) == E4M3_MAX
    # relative error of each element: at most half a unit in the last place of its binade (2^-4),
    # plus the subnormal floor (2^-10 of the row's scale)
    err = np.abs(deq[rows] - x[rows])
    bound = np.abs(x[rows]) * 2.0 ** -4 + 2.0 ** -10 * s[rows, None]
    assert np.all(err <= bound * (1 + 1e-6))


def test_gemm_fp8_equals_product_of_torch_decoded_operands():
    rng = np.random.default_rng(5)
    a = rng.integers(0, 256, (37, 96), dtype=np.uint8)
    w = rng.integers(0, 256, (29, 96), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x10                 # no NaN codes
    w[(w & 0x7F) == 0x7F] = 0x10
    sa = rng.uniform(0.5, 2, 37).astype(np.float32)
    sw = rng.uniform(0.5, 2, 29).astype(np.float32)
    ref = (_torch_decode(a).astype(np.float64) @ _torch_decode(w).astype(np.float64).T) \
        * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    np.testing.assert_allclose(gemm_fp8(a, sa, w, sw), ref, rtol=1e-13, atol=0)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.standard_normal(200000) * 10, rng.standard_normal(1000) * 1e-30,
                        np.float32([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 3.0e38])]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(bf16_round_f32(x), ref)


# ---- FP8 attention ---------------------------------------------------------------------
from oracle.attention import block_causal_attention
from oracle.fp8 import P_BIAS, attention_fp8

LOG2E = float(np.log2(np.e))


def _exact_attention(q_codes, k_codes, v_codes, sq, sk, sv):
    """Softmax attention of the dequantized operands (the plain oracle, fp64)."""
    q = e4m3_decode(q_codes) * np.asarray(sq, np.float64)[None, :, None]
    k = e4m3_decode(k_codes) * np.asarray(sk, np.float64)[None, :, None]
    v = e4m3_decode(v_codes) * np.asarray(sv, np.float64)[None, :, None]
    return block_causal_attention(q, {0: (k, v)}, None, qblock=0, window=0)


def _gauss_codes(rng, shape, sigma=1.0):
    return e4m3_encode((rng.standard_normal(shape) * sigma).astype(np.float32))


def test_attention_fp8_is_exact_softmax_attention_when_p_is_a_power_of_two():
    """Scores that are whole numbers in the log2 domain make every P = 2^(s - M + bias) a
    power of two within e4m3's normal range, so its rounding is exact and the FP8 result
    must equal plain softmax attention of the dequantized operands."""
    rng = np.random.default_rng(11)
    T, N, H, d = 6, 40, 2, 16
    q = np.zeros((T, H, d), np.uint8)
    k = np.zeros((N, H, d), np.uint8)
    q[:, :, 0] = e4m3_encode(rng.choice([1.0, 2.0], size=(T, H)).astype(np.float32))
    k[:, :, 0] = e4m3_encode(rng.integers(-4, 3, size=(N, H)).astype(np.float32))
    v = _gauss_codes(rng, (N, H, d))
    sq = np.float32([1.0, 0.5])
    # q_scale * k_scale * log2(e) / sqrt(d) = 1 up to the float32 rounding of k_scale
    sk = (np.float32(np.sqrt(d) / LOG2E) / sq).astype(np.float32)
    sv = np.float32([0.25, 3.0])
    got = attention_fp8(q, k, v, sq, sk, sv)
    ref = _exact_attention(q, k, v, sq, sk, sv)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-7 * np.abs(ref).max())


def test_attention_fp8_single_key_returns_its_value():
    rng = np.random.default_rng(12)
    q = _gauss_codes(rng, (5, 1, 32))
    k = _gauss_codes(rng, (1, 1, 32))
    v = _gauss_codes(rng, (1, 1, 32))
    # P of the lone key is 2^(s - ceil(s) + bias), rounded to e4m3 in the product but not
    # in the normaliser: the output is v times that rounding ratio, within 2^-4 of 1
    got = attention_fp8(q, k, v, [1.0], [1.0], [2.0])
    s = (e4m3_decode(q[:, 0]) @ e4m3_decode(k[:, 0]).T) / np.sqrt(32) * LOG2E
    p = np.exp2(s - np.ceil(s) + P_BIAS).astype(np.float32)
    ratio = e4m3_decode(e4m3_encode(p)) / p.astype(np.float64)
    np.testing.assert_allclose(got[:, 0, :], ratio * 2.0 * e4m3_decode(v[0, 0])[None, :], rtol=1e-12)
    assert np.all(np.abs(ratio - 1) <= 2.0 ** -4)


def test_attention_fp8_is_unchanged_by_a_whole_number_shift_of_all_scores():
    """Adding the same whole number to every score of a row moves M by it and scales
    every P by a power of two, which e4m3 represents exactly in its normal range."""
    rng = np.random.default_rng(13)
    T, N, H, d = 8, 64, 1, 16
    q = _gauss_codes(rng, (T, H, d), 0.5)
    k = _gauss_codes(rng, (N, H, d), 0.5)
    v = _gauss_codes(rng, (N, H, d))
    q[:, :, d - 1] = e4m3_encode([1.0])[0]
    sq = np.float32([1.0])
    sk = np.float32([np.sqrt(d) / LOG2E])
    outs = []
    for shift in (0.0, 3.0, -5.0):
        kk = k.copy()
        kk[:, :, d - 1] = e4m3_encode([shift])[0]
        outs.append(attention_fp8(q, kk, v, sq, sk, [1.0]))
    np.testing.assert_allclose(outs[1], outs[0], rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(outs[2], outs[0], rtol=1e-5, atol=1e-9)


def test_attention_fp8_error_is_within_the_rounding_bound_of_p():
    """Against softmax attention of the dequantized operands, the only rounding is P's:
    at most half an e4m3 unit (2^-4 relative) for normal values, and half the
    subnormal step (2^-10) below 2^-6, against a normaliser of at least 2^(bias-1)."""
    rng = np.random.default_rng(14)
    T, N, H, d = 40, 300, 2, 64
    q = _gauss_codes(rng, (T, H, d))
    k = _gauss_codes(rng, (N, H, d))
    v = _gauss_codes(rng, (N, H, d))
    for i in range(8):                          # rows dominated by one key
        j = int(rng.integers(N))
        q[i] = e4m3_encode(e4m3_decode(k[j]).astype(np.float32) * 2.0)
    sq, sk, sv = np.float32([1.0, 0.5]), np.float32([0.5, 1.0]), np.float32([1.0, 2.0])
    got = attention_fp8(q, k, v, sq, sk, sv)
    ref = _exact_attention(q, k, v, sq, sk, sv)
    qd = e4m3_decode(q) * sq[None, :, None]
    kd = e4m3_decode(k) * sk[None, :, None]
    vd = np.abs(e4m3_decode(v) * sv[None, :, None])
    for h in range(H):
        s = qd[:, h] @ kd[:, h].T / np.sqrt(d)
        w = np.exp(s - s.max(axis=1, keepdims=True))
        w /= w.sum(axis=1, keepdims=True)
        bound = np.maximum(2.0 ** -4 * w, 2.0 ** -10 / 2.0 ** (P_BIAS - 1)) @ vd[:, h]
        assert np.all(np.abs(got[:, h] - ref[:, h]) <= bound * (1 + 1e-6) + 1e-12)
    # the rounding of P is visible: the result is not the unquantized one
    assert np.abs(got - ref).max() > 1e-4 * np.abs(ref).max()


# ---- e4m3 attention operands of the stream ---------------------------------------------------
from oracle.fp8 import ATTN_ACT_BOUND, attn_fp8_scales, pow2_at_least, quantize_heads  # noqa: E402
from oracle.norm import rms_norm  # noqa: E402
from oracle.rope import rope_rotate  # noqa: E402


def test_pow2_at_least():
    assert [pow2_at_least(x) for x in (1.0, 1.5, 0.75, 2.0 ** -10, 3 * 2.0 ** -10, 448.0)] == \
        [1.0, 2.0, 1.0, 2.0 ** -10, 2.0 ** -8, 512.0]


def test_quantize_heads_is_torch_e4m3_of_value_over_scale():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((50, 3, 16)) * 20
    sc = np.float32([0.5, 1.0, 0.125])
    got = quantize_heads(x, sc)
    ref = (torch.from_numpy(x.astype(np.float32)) / torch.from_numpy(sc)[None, :, None]) \
        .clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, ref)


def _adversarial_inputs(w, D, rows):
    """Unit-RMS rows aligned with weight rows (or sums of a rotary pair of rows), the
    inputs that come closest to the Cauchy-Schwarz bound."""
    xs = []
    for r in rows:
        x = w[r] if r % 2 else w[r] + w[r + 1]
        xs.append(x / np.sqrt(np.mean(x ** 2)))
    return np.stack(xs)


def test_attn_fp8_scales_never_saturate_and_are_tight():
    rng = np.random.default_rng(22)
    D, H, d = 256, 4, 64
    w = (rng.standard_normal((3 * D, D)) * rng.uniform(0.2, 3.0, (3 * D, 1)) * 0.02)
    sc = attn_fp8_scales(w, D, H, d).astype(np.float64)
    assert np.all(np.log2(sc) == np.round(np.log2(sc)))          # powers of two
    # random and adversarial unit-RMS rows, rounded up by the largest operand rounding (6.25 %)
    x = np.concatenate([rms_norm(rng.standard_normal((200, D))),
                        _adversarial_inputs(w, D, rng.integers(0, 3 * D - 1, 300))]) * (1 + 2.0 ** -4)
    qkv = x @ w.T
    pairs = (d // 2 - 2 * (d // 6), d // 6, d // 6)
    pos = [rng.integers(-50, 50, len(x)) for _ in range(3)]
    for part in range(3):
        vals = qkv[:, part * D:(part + 1) * D].reshape(len(x), H, d)
        if part < 2:
            vals = rope_rotate(vals, *pos, pairs, 10000.0)
        ratio = np.abs(vals).max(axis=(0, 2)) / sc[part]
        assert np.all(ratio <= 448.0), (part, ratio)
    # the bound itself lands in (224, 448] of each head's scale
    n2 = (w ** 2).sum(axis=1)
    for part in range(3):
        for h in range(H):
            rows = n2[part * D + h * d: part * D + (h + 1) * d]
            m = (rows[0::2] + rows[1::2]).max() if part < 2 else rows.max()
            b = ATTN_ACT_BOUND * np.sqrt(D * m) / sc[part, h]
            assert 224.0 < b <= 448.0


def test_attn_fp8_scales_pair_bound_is_needed_for_rotated_rows():
    """A rotation by 45 degrees of a pair whose rows both read the input puts sqrt(2)
    times a row's bound into one component: the pair norm is what bounds it."""
    D, H, d = 16, 1, 16
    w = np.zeros((3 * D, D))
    w[0, 0] = w[1, 0] = 1.0                      # q rows 0 and 1 (rotary pair 0) read input 0
    w[D:, :] = 0.01
    x = np.zeros((1, D))
    x[0, 0] = np.sqrt(D)                         # unit RMS
    q = (x @ w[:D].T).reshape(1, H, d)
    # pair 0 is temporal with frequency 1: angle = position = pi/4
    qr = rope_rotate(q, np.array([np.pi / 4]), np.array([0]), np.array([0]), (d // 2, 0, 0), 10000.0)
    v = abs(qr[0, 0, 1])
    assert v == pytest.approx(np.sqrt(2) * np.sqrt(D))
    assert v > ATTN_ACT_BOUND * np.sqrt(D) * 1.0                 # above the bound of a single row
    assert v <= ATTN_ACT_BOUND * np.sqrt(D) * np.sqrt(2.0)       # within the pair's bound
    assert v / attn_fp8_scales(w, D, H, d)[0, 0] <= 448.0


def test_oracle_stream_with_e4m3_attention_stays_near_the_exact_stream():
    """The e4m3 attention changes the finished latents only by the format's rounding
    (a few per cent on this flat-attention synthetic stack), block by block."""
    from oracle import OracleStream
    from workloads import DTYPE_BF16, SINK_AAS, StreamConfig, Workload, block_noise, make_weights
    cfg = StreamConfig(num_layers=2, hidden=256, heads=2, head_dim=128, latent_ch=32, grid_h=4, grid_w=6,
                       window_blocks=2, sink_mode=SINK_AAS, dtype=DTYPE_BF16, attn_fp8=1)
    wl = Workload("afp8", cfg, 5, 4, 1.5 / 16.0, 0.1)
    W = make_weights(wl)
    o8, o = OracleStream(cfg, W), OracleStream(cfg.replace(attn_fp8=0), W)
    o8.set_sink(W.sink)
    o.set_sink(W.sink)
    for k in range(wl.num_blocks + 3):
        xn = block_noise(wl, k) if k < wl.num_blocks else None
        a, fa = o8.denoise_step(xn)
        b, fb = o.denoise_step(xn)
        assert fa == fb
        if fa >= 0:
            rel = np.abs(a - b).sum() / np.abs(b).sum()
            assert 1e-3 < rel < 0.08, (fa, rel)
