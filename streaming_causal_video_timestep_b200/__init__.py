"""B200-native timestep-forced streaming denoising step (Live Avatar's streaming DiT step).

The product is the C-ABI library libla.so (include/la_stream.h) built from
csrc/ for sm_100a; this package is its thin Python binding.  Importing the
package does not load the library; LaStream / op_* load it and raise if it
has not been built (there is no CPU fallback).
"""
from ._lib import LaError, exported_symbols, load  # noqa: F401


def __getattr__(name):
    if name in ("LaStream", "op_gemm", "op_attention", "op_euler", "op_quantize_e4m3", "op_gemm_fp8",
                "op_attention_fp8", "torch_dtype", "sched_trace"):
        from . import stream
        return getattr(stream, name)
    raise AttributeError(name)
