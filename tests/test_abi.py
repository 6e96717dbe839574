"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument checks return their status codes without touching a GPU."""
import ctypes
import os
import re

import pytest

import streaming_causal_video_timestep_b200 as pkg
from streaming_causal_video_timestep_b200 import _lib
from workloads import TINY, make_weights

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(la_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from streaming_causal_video_timestep_b200 import build
    build.build()
    return _lib.load()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert len(declared) >= 19
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(_lib.exported_symbols()) == declared


def test_status_strings(lib):
    assert lib.la_status_string(0) == b"ok"
    assert lib.la_status_string(-1) == b"invalid argument"
    assert lib.la_status_string(-5) == b"device error"
    assert lib.la_status_string(7) == b"unknown status"
    assert lib.la_last_error(None) == b"no stream"


def test_destroy_null_is_noop(lib):
    assert lib.la_stream_destroy(None) == 0


def _cfg(**over):
    base = dict(num_layers=1, hidden=64, heads=1, head_dim=64, latent_ch=64, grid_h=4, grid_w=4,
                frames_per_block=3, sink_frames=1, window_blocks=2, num_steps=4, rope_split=(12, 10, 10),
                rope_theta=10000.0, sink_mode=1, rolling_rope=1, sink_offset_frames=3, schedule=0, dtype=1)
    base.update(over)
    ts = over.pop("timesteps", (1.0, 0.75, 0.5, 0.25, 0.0))
    c = _lib.LaConfig()
    for k, v in base.items():
        if k == "rope_split":
            c.rope_split = (ctypes.c_int32 * 3)(*v)
        elif k != "timesteps":
            setattr(c, k, v)
    arr = (ctypes.c_float * len(ts))(*ts)
    c.timesteps = ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
    c._keep = arr
    return c


def _weights(nonnull=True):
    w = _lib.LaWeights()
    arr = (ctypes.c_void_p * 1)(0x1000 if nonnull else 0)
    w.w_qkv = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    w.w_out = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    w._keep = arr
    return w


@pytest.mark.parametrize("over", [
    dict(num_layers=0), dict(hidden=-64), dict(heads=2), dict(head_dim=60, hidden=60),
    dict(dtype=0),                                    # bf16 needs head_dim 128
    dict(timesteps=(1.0, 0.5, 0.75, 0.25, 0.0)),      # not descending
    dict(timesteps=(1.0, 0.75, 0.75, 0.25, 0.0)),     # not strictly
    dict(window_blocks=-1), dict(window_blocks=15), dict(rope_split=(10, 10, 10)),
    dict(sink_frames=2), dict(num_steps=0, timesteps=(1.0,)), dict(num_steps=9),
    dict(sink_mode=5), dict(schedule=3), dict(rope_theta=0.0), dict(frames_per_block=0),
    dict(latent_ch=32),                               # identity needs latent_ch == hidden
    dict(cache_mode=2),
    dict(cache_mode=1, schedule=0),                   # the clean-cache refresh is sequential only
    dict(proj_fp8=1),                                 # e4m3 projections need the bf16 stream (dtype 1 = fp32)
    dict(proj_fp8=2, dtype=0, head_dim=128, hidden=128, latent_ch=128, rope_split=(22, 21, 21)),
    dict(attn_fp8=1),                                 # e4m3 attention needs the bf16 stream
    dict(cache_mode=2, schedule=0),                   # the fixed-noise cache is sequential only
    dict(cache_mode=2, schedule=1, cache_step=4),     # cache_step names a step
    dict(cache_mode=3),
    dict(schedule=2, slot_index=4),                   # slot_index names a step
    dict(schedule=2, slot_index=0, cache_mode=1),     # a slot stream keeps its own step's cache
    dict(attn_fp8=2, dtype=0, head_dim=128, hidden=128, latent_ch=128, rope_split=(22, 21, 21)),
])
def test_invalid_config_returns_einval(lib, over):
    c = _cfg(**over)
    h = ctypes.c_void_p()
    code = lib.la_stream_create(ctypes.byref(c), ctypes.byref(_weights()), None, ctypes.byref(h))
    assert code == _lib.LA_EINVAL
    assert not h.value


def test_null_weights_return_einval(lib):
    h = ctypes.c_void_p()
    assert lib.la_stream_create(ctypes.byref(_cfg()), ctypes.byref(_weights(False)), None,
                                ctypes.byref(h)) == _lib.LA_EINVAL
    assert lib.la_stream_create(ctypes.byref(_cfg()), None, None, ctypes.byref(h)) == _lib.LA_EINVAL
    assert lib.la_stream_create(None, None, None, None) == _lib.LA_EINVAL


def test_null_stream_calls_return_einval(lib):
    fin = ctypes.c_int64()
    assert lib.la_denoise_step(None, None, None, ctypes.byref(fin)) == _lib.LA_EINVAL
    assert lib.la_set_sink(None, None) == _lib.LA_EINVAL
    assert lib.la_synchronize(None) == _lib.LA_EINVAL
    assert lib.la_index_state_size(None) == 0
    assert lib.la_launch_count(None) == 0


def test_op_entry_points_reject_bad_sizes(lib):
    assert lib.la_op_gemm(0, 0, None, None, None, None, 0, 0, 0, None, 0, None) == _lib.LA_EINVAL
    assert lib.la_op_euler(None, None, 0, 0, None, 0, None) == _lib.LA_EINVAL
    assert lib.la_op_attention(0, None, 0, 0, 0, 0, None, None, None, None, None, 0, None) == _lib.LA_EINVAL
    # FP8 attention: NULL pointers, and head_dim other than 128 with every pointer set
    assert lib.la_op_attention_fp8(None, 0, 0, 0, 0, None, None, None, None, None, None, None, None,
                                   None) == _lib.LA_EINVAL
    buf = ctypes.c_void_p(16)
    ptrs = (ctypes.c_void_p * 1)(16)
    lens = (ctypes.c_int64 * 1)(128)
    assert lib.la_op_attention_fp8(buf, 128, 1, 64, 1, ptrs, ptrs, lens, buf, buf, buf, buf, None,
                                   None) == _lib.LA_EINVAL
    lens0 = (ctypes.c_int64 * 1)(0)
    assert lib.la_op_attention_fp8(buf, 128, 1, 128, 1, ptrs, ptrs, lens0, buf, buf, buf, buf, None,
                                   None) == _lib.LA_EINVAL


def test_valid_config_without_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    code = lib.la_stream_create(ctypes.byref(_cfg()), ctypes.byref(_weights()), None, ctypes.byref(h))
    assert code == _lib.LA_ECUDA and not h.value


def test_package_import_does_not_route_through_the_oracle():
    import sys
    assert "oracle" not in {m.split(".")[0] for m in pkg.__dict__.get("__all__", [])}
    src_dir = os.path.dirname(pkg.__file__)
    for root, _, files in os.walk(src_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cpp", ".h", ".cuh")):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
