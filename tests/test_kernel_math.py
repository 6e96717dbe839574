"""Host-side checks of the arithmetic the attention kernel uses in place of ex2.

The softmax of the tcgen05 attention kernel computes part of its
exponentials 2^x on the FMA pipe (exp2_poly2 in csrc/attn_tc.cu): clamp at
-125, split x = j + f with j = round(x) through the 1.5 * 2^23 shifter, a
degree-3 polynomial p(f) with p(0) = 1 for 2^f on [-1/2, 1/2], and j added to
the exponent field.  These tests replay those steps in numpy float32 with the
constants read from the kernel source, and check them against the
mathematics: the relative error bound over the whole input range, exact powers
of two at integer inputs, and monotone, finite output.  The GPU parity tests of
the attention op check the device code itself.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(__file__), "..", "streaming_causal_video_timestep_b200", "csrc", "attn_tc.cu")
REL_BOUND = 1.02e-4          # the fit's maximum relative error on [-1/2, 1/2]
BF16_HALF_ULP = 2.0 ** -9    # relative rounding bound of bf16 (8 significant bits)


def _constants():
    text = open(SRC).read()
    m = re.search(r"c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f", text)
    assert m, "polynomial constants not found in the kernel source"
    return [np.float32(float(v)) for v in m.groups()]


def exp2_poly(x):
    """The kernel's steps, one float32 rounding per step (fma rounds once)."""
    c1, c2, c3 = _constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    j = (t - shift).astype(np.float32)
    f = (x - j).astype(np.float32)                       # exact
    f64 = f.astype(np.float64)
    p = np.float32(f64 * np.float64(c3) + np.float64(c2))   # fma: exact product, one rounding
    p = np.float32(p.astype(np.float64) * f64 + np.float64(c1))
    p = np.float32(p.astype(np.float64) * f64 + 1.0)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_fraction_split_is_exact_and_in_range():
    x = np.linspace(-125.0, 9.0, 200001, dtype=np.float32)
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    j = (t - shift).astype(np.float32)
    f = (x - j).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    assert np.all(j == np.round(x.astype(np.float64)))   # round half to even, like the fp32 add
    assert np.all(f.astype(np.float64) + j.astype(np.float64) == x.astype(np.float64))


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-125.0, 9.0, 400001), rng.uniform(-30.0, 0.0, 400000)]).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert np.isfinite(got).all() and (got > 0).all()
    assert rel.max() <= REL_BOUND, rel.max()
    assert rel.max() < BF16_HALF_ULP / 15


def test_integer_inputs_give_exact_powers_of_two():
    k = np.arange(-125, 9, dtype=np.float32)
    assert np.array_equal(exp2_poly(k), np.exp2(k.astype(np.float64)).astype(np.float32))
    assert exp2_poly(np.float32(0.0)) == np.float32(1.0)   # the row maximum contributes exactly 1


def test_clamp_keeps_very_negative_inputs_tiny_and_normal():
    x = np.array([-125.0, -126.5, -1e4, -np.inf], np.float32)
    y = exp2_poly(x)
    assert np.all(y == np.float32(2.0 ** -125))
    assert np.all(y >= np.finfo(np.float32).tiny)


def test_monotone_on_a_fine_grid():
    x = np.linspace(-20.0, 8.0, 100001, dtype=np.float32)
    y = exp2_poly(x)
    assert np.all(np.diff(y.astype(np.float64)) >= 0)
