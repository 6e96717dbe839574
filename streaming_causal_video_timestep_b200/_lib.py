"""ctypes declarations of the C ABI in include/la_stream.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla.so")

LA_OK, LA_EINVAL, LA_ESTATE, LA_ENOMEM, LA_ECUDA, LA_EDEVICE = 0, -1, -2, -3, -4, -5
LA_SINK_FIXED, LA_SINK_AAS = 0, 1
LA_SCHED_PIPELINED, LA_SCHED_SEQUENTIAL = 0, 1
LA_BF16, LA_FP32 = 0, 1
LA_MAX_STEPS, LA_MAX_WINDOW, LA_MAX_FPB = 8, 14, 7
LA_EPI_STORE, LA_EPI_RESID, LA_EPI_SET32, LA_EPI_EULER, LA_EPI_STORE32 = 0, 1, 2, 3, 4

TAP = dict(x_in=0, x_out=1, h=2, q=3, o=4, v=5, ring_k=6, ring_v=7, sink_k=8, sink_v=9, sink_k_rope=10, sink_h=11,
           hop=12, sink_hop=13, sink_v8=14, attn_scales=15, h_mid=16, ffn_u=17, h_cross=18, xq=19, xk=20, xv=21,
           xo=22)
KIND = dict(in_proj=0, qkv_gemm=1, rope=2, attn=3, out_gemm=4, head=5, other=6, ffn=7, cross=8)


class LaConfig(ctypes.Structure):
    _fields_ = [
        ("num_layers", c_int32), ("hidden", c_int32), ("heads", c_int32), ("head_dim", c_int32),
        ("latent_ch", c_int32), ("grid_h", c_int32), ("grid_w", c_int32), ("frames_per_block", c_int32),
        ("sink_frames", c_int32), ("window_blocks", c_int32), ("num_steps", c_int32),
        ("timesteps", POINTER(c_float)), ("rope_split", c_int32 * 3), ("rope_theta", c_double),
        ("sink_mode", c_int32), ("rolling_rope", c_int32), ("sink_offset_frames", c_int32),
        ("schedule", c_int32), ("dtype", c_int32), ("cache_mode", c_int32), ("proj_fp8", c_int32),
        ("attn_fp8", c_int32), ("cache_step", c_int32), ("block_kind", c_int32), ("ffn_dim", c_int32),
        ("audio_tokens", c_int32), ("audio_dim", c_int32), ("slot_index", c_int32),
    ]


class LaWeights(ctypes.Structure):
    _fields_ = [("w_in", c_void_p), ("w_head", c_void_p), ("w_qkv", POINTER(c_void_p)),
                ("w_out", POINTER(c_void_p)), ("w_ffn1", POINTER(c_void_p)), ("w_ffn2", POINTER(c_void_p)),
                ("ada", c_void_p), ("w_qc", POINTER(c_void_p)), ("w_kvc", POINTER(c_void_p)),
                ("w_oc", POINTER(c_void_p))]


class LaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{msg} (status {code})")
        self.code = code


_lib = None


def load():
    """Load libla.so; raises if it is missing (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} not built: run python -m streaming_causal_video_timestep_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "la_stream_create": (c_int, [POINTER(LaConfig), POINTER(LaWeights), c_void_p, POINTER(c_void_p)]),
        "la_set_sink": (c_int, [c_void_p, c_void_p]),
        "la_denoise_step": (c_int, [c_void_p, c_void_p, c_void_p, POINTER(c_int64)]),
        "la_denoise_step_av": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, POINTER(c_int64)]),
        "la_replace_sink": (c_int, [c_void_p, c_void_p]),
        "la_denoise_step_host": (c_int, [c_void_p, c_void_p, c_void_p, POINTER(c_int64)]),
        "la_synchronize": (c_int, [c_void_p]),
        "la_stream_destroy": (c_int, [c_void_p]),
        "la_last_error": (c_char_p, [c_void_p]),
        "la_status_string": (c_char_p, [c_int]),
        "la_index_state_size": (c_int64, [c_void_p]),
        "la_get_index_state": (c_int, [c_void_p, POINTER(c_int32), c_int64]),
        "la_sched_state_size": (c_int64, [c_void_p]),
        "la_sched_trace": (c_int, [c_void_p, c_int32, c_void_p, POINTER(c_int32), c_int64]),
        "la_debug_capture": (c_int, [c_void_p, c_int32]),
        "la_debug_tap": (c_int, [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_int64]),
        "la_debug_set_slot_input": (c_int, [c_void_p, c_int32, c_void_p]),
        "la_profile_enable": (c_int, [c_void_p, c_int32]),
        "la_profile_read": (c_int, [c_void_p, c_int32, POINTER(c_int64), POINTER(c_double)]),
        "la_launch_count": (c_int64, [c_void_p]),
        "la_op_gemm": (c_int, [c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                               c_int64, POINTER(c_float), c_int64, c_void_p]),
        "la_op_attention": (c_int, [c_int32, c_void_p, c_int64, c_int32, c_int32, c_int32, POINTER(c_void_p),
                                    POINTER(c_void_p), POINTER(c_int64), c_void_p, c_void_p, c_int32, c_void_p]),
        "la_op_euler": (c_int, [c_void_p, c_void_p, c_int64, c_int64, POINTER(c_float), c_int64, c_void_p]),
        "la_op_attention_static": (c_int, [c_void_p, c_int64, c_int32, c_int32, c_int32, POINTER(c_void_p),
                                           POINTER(c_void_p), POINTER(c_int64), c_void_p, c_void_p, c_void_p]),
        "la_debug_wait_timeout": (c_int, [c_int64, c_int32, POINTER(c_int32)]),
        "la_debug_op_wait_timeout": (c_int, [c_int64, c_void_p]),
        "la_op_status": (c_int, [c_void_p]),
        "la_op_quantize_e4m3": (c_int, [c_int32, c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
        "la_op_gemm_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_int64, c_int64,
                                   c_int64, c_void_p]),
        "la_op_attention_fp8": (c_int, [c_void_p, c_int64, c_int32, c_int32, c_int32, POINTER(c_void_p),
                                        POINTER(c_void_p), POINTER(c_int64), c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def exported_symbols():
    """Names of the C-ABI functions declared in include/la_stream.h."""
    return [
        "la_stream_create", "la_set_sink", "la_denoise_step", "la_denoise_step_host", "la_denoise_step_av",
        "la_replace_sink",
        "la_synchronize",
        "la_stream_destroy", "la_last_error", "la_status_string", "la_index_state_size", "la_get_index_state",
        "la_debug_capture", "la_debug_tap", "la_debug_set_slot_input", "la_profile_enable", "la_profile_read",
        "la_launch_count", "la_op_gemm", "la_op_attention", "la_op_euler", "la_op_attention_static",
        "la_debug_wait_timeout", "la_op_quantize_e4m3", "la_op_gemm_fp8", "la_op_attention_fp8",
        "la_debug_op_wait_timeout", "la_op_status", "la_sched_state_size", "la_sched_trace",
    ]


def check(code, handle=None):
    if code != LA_OK:
        lib = load()
        msg = lib.la_last_error(handle).decode() if handle else lib.la_status_string(code).decode()
        raise LaError(code, msg or lib.la_status_string(code).decode())
