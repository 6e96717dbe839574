"""bench.py's per-kernel table, on the host: the figures it derives from the
library's profiling counters (launches and total milliseconds per kernel kind).

The counters below are those of a bench run of the 8-sublayer, 4-slot stream
at the 14B-like shape on a B200 (10 timed ticks); the expected TFLOP/s and
GB/s are the ones that run printed.  They are recomputed here from the stated
FLOP and byte counts, so a wrong count or unit shows up as a mismatch.
"""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

SHAPE = dict(L=8, S=4, T=4680, D=5120, C=64, F=1560)
PEAKS = {"tflops": 1628.9, "tflops_sust": 1376.3, "hbm": 6538.6, "src": "measured"}
# kind: (launches, average ms) over 10 ticks, and the figure the run printed
RUN = {
    "in_proj": (20, 0.1219, 100.6),
    "qkv_gemm": (80, 2.0066, 1467.4),
    "rope": (80, 0.0253, 3784.8),
    "attn": (80, 5.8718, 1018.6),
    "out_gemm": (80, 0.7291, 1346.2),
    "head": (10, 0.0485, 253.0),
    "other": (100, 0.1041, None),
}


def _table(run=RUN, steps=10):
    kinds = {k: (n, n * avg) for k, (n, avg, _) in run.items()}
    return bench.kernel_entries(kinds, steps, attn_tflops=RUN["attn"][2], pk=PEAKS, **SHAPE)


def test_tensor_kinds_reproduce_the_printed_tflops_and_carry_the_peak_fraction():
    tab = _table()
    for kind in ("in_proj", "qkv_gemm", "attn", "out_gemm", "head"):
        want = RUN[kind][2]
        # the run rounded ms_avg to 4 decimals before printing it
        assert tab[kind]["tflops"] == pytest.approx(want, rel=2e-3), kind
        assert tab[kind]["frac_sustained"] == pytest.approx(tab[kind]["tflops"] / PEAKS["tflops_sust"], abs=1e-3)
    # QKV: 2 * (4 slots x 4680 tokens) * 5120 * 15360 FLOP per launch
    assert 2.0 * 4 * 4680 * 5120 * 15360 / 2.0066e-3 / 1e12 == pytest.approx(tab["qkv_gemm"]["tflops"], abs=0.2)


def test_rope_reports_bandwidth_against_the_measured_copy():
    tab = _table()
    e = tab["rope"]
    # read the fp32 un-roped sink K once, write 4 bf16 roped copies
    assert e["bytes_per_launch"] == 1560 * 5120 * 4 + 4 * 1560 * 5120 * 2
    assert e["gbs"] == pytest.approx(RUN["rope"][2], rel=2e-3)
    assert e["frac_hbm"] == pytest.approx(e["gbs"] / PEAKS["hbm"], abs=1e-3)
    assert "tflops" not in e and "frac_sustained" not in e


def test_other_kinds_and_partial_counts():
    tab = _table()
    assert set(tab["other"]) == {"launches", "ms_avg", "ms_per_step"}
    assert tab["attn"]["ms_per_step"] == pytest.approx(80 * 5.8718 / 10, abs=1e-3)
    # a kind that never launched is left out
    run = dict(RUN, head=(0, 0.0485, None))
    assert "head" not in _table(run)
    # a GEMM kind with fewer launches than one a layer and tick gets no FLOP rate
    run = dict(RUN, out_gemm=(40, 0.7291, None))
    assert "tflops" not in _table(run)["out_gemm"]


def test_rope_launch_covering_every_layer_counts_every_layers_bytes():
    """One sink re-rope launch a tick for all 8 layers: 8x the bytes of a per-layer launch."""
    run = dict(RUN, rope=(10, 0.1300, None))
    e = _table(run)["rope"]
    assert e["bytes_per_launch"] == 8 * (1560 * 5120 * 4 + 4 * 1560 * 5120 * 2)
    assert e["gbs"] == pytest.approx(e["bytes_per_launch"] / 0.1300e-3 / 1e9, rel=1e-3)
