"""The allocation-free attention entry point (la_op_attention_static).

Callers that cannot allocate device memory (plugins whose host application
owns all device memory, real-time paths) use this variant: its scratch -- the scaled queries the attention kernel
reads -- lives in a static device array inside the library.  This test calls it
through the C ABI twice in a row, with different inputs and sizes, and checks
each output against the fp64 oracle's block-causal attention (sink + two
blocks, all visible) at the bf16 tolerance, and against the allocating entry
point la_op_attention given the same
query already scaled (q_scaled=1, q*log2(e)/sqrt(d) rounded once to bf16), with
the tolerance the other GPU tests use; both run the same attention kernel on the
same bf16 operands, so the outputs also agree bit for bit.  The file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

from oracle import block_causal_attention
from workloads import DTYPE_BF16, bf16_round, random_array

from _helpers import assert_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

STATIC_Q_ELEMS = 8 * 1024 * 1024     # LA_STATIC_Q_ELEMS in include/la_stream.h
SCALE_LOG2 = float(np.float32(1.4426950408889634 / np.sqrt(128.0)))   # log2(e)/sqrt(d) as fp32


@pytest.fixture(scope="module")
def lib():
    from streaming_causal_video_timestep_b200 import _lib, build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return _lib.load()


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(bf16_round(a))).cuda().to(torch.bfloat16)


def _segments(ks, vs):
    n = len(ks)
    kp = (ctypes.c_void_p * n)(*[k.data_ptr() for k in ks])
    vp = (ctypes.c_void_p * n)(*[v.data_ptr() for v in vs])
    ln = (ctypes.c_int64 * n)(*[k.shape[1] for k in ks])
    return n, kp, vp, ln


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_static_scratch_attention_matches_allocating_entry_point_twice(lib):
    H, d, F, T = 3, 128, 60, 180
    for call, (seed, Tq) in enumerate(((1, 300), (2, 180))):   # the second call uses less of the array
        q = _bf16(random_array(seed, (H, Tq, d)))
        q_scaled = (q.float() * SCALE_LOG2).to(torch.bfloat16)   # fp32 product, one rounding
        ks = [_bf16(random_array(seed + 10 + i, (H, n, d))) for i, n in enumerate((F, T, T))]
        vs = [_bf16(random_array(seed + 20 + i, (H, n, d))) for i, n in enumerate((F, T, T))]
        n, kp, vp, ln = _segments(ks, vs)
        ref = torch.empty((Tq, H * d), dtype=torch.bfloat16, device="cuda")
        ref32 = torch.empty((Tq, H * d), dtype=torch.float32, device="cuda")
        got = torch.empty_like(ref)
        got32 = torch.empty_like(ref32)
        assert lib.la_op_attention(0, ctypes.c_void_p(q_scaled.data_ptr()), Tq, H, d, n, kp, vp, ln,
                                   ctypes.c_void_p(ref.data_ptr()), ctypes.c_void_p(ref32.data_ptr()), 1,
                                   _stream()) == 0
        assert lib.la_op_attention_static(ctypes.c_void_p(q.data_ptr()), Tq, H, d, n, kp, vp, ln,
                                          ctypes.c_void_p(got.data_ptr()), ctypes.c_void_p(got32.data_ptr()),
                                          _stream()) == 0
        torch.cuda.synchronize()
        assert lib.la_op_status(_stream()) == 0, f"call {call}: a kernel reported a device error"
        # against the fp64 oracle's block-causal attention on the operands the kernel
        # reads: the query it consumes is q * log2(e)/sqrt(d) rounded once to bf16,
        # i.e. the query q_scaled / (log2(e)/sqrt(d)) in the oracle's natural-log form
        hm = lambda t: t.double().cpu().numpy().transpose(1, 0, 2)         # [H, n, d] -> [n, H, d]
        want = block_causal_attention(hm(q_scaled) / SCALE_LOG2, {0: (hm(ks[1]), hm(vs[1])),
                                                                   1: (hm(ks[2]), hm(vs[2]))},
                                      (hm(ks[0]), hm(vs[0])), qblock=1, window=1).reshape(Tq, H * d)
        assert_close(got32.cpu().numpy(), want, DTYPE_BF16, f"call {call}: fp32 output against the oracle")
        assert_close(got32.cpu().numpy(), ref32.cpu().numpy(), DTYPE_BF16, f"call {call}: fp32 output")
        assert_close(got.float().cpu().numpy(), ref.float().cpu().numpy(), DTYPE_BF16, f"call {call}: bf16 output")
        assert torch.equal(got32, ref32) and torch.equal(got, ref), f"call {call}: not bitwise equal"


def test_static_scratch_rejects_sizes_beyond_the_array(lib):
    from streaming_causal_video_timestep_b200 import _lib
    H, d = 40, 128
    Tq = STATIC_Q_ELEMS // (H * d) + 1
    q = torch.empty((H, Tq, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((H, 16, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((Tq, H * d), dtype=torch.bfloat16, device="cuda")
    n, kp, vp, ln = _segments([k], [k])
    code = lib.la_op_attention_static(ctypes.c_void_p(q.data_ptr()), Tq, H, d, n, kp, vp, ln,
                                      ctypes.c_void_p(out.data_ptr()), None, _stream())
    assert code == _lib.LA_EINVAL
