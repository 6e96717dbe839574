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
