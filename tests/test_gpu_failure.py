"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up after its limit, raises the device error word and returns;
the host reads LA_EDEVICE and the context stays usable.  The op-level entry
points report through their own word, read and cleared by la_op_status."""
import ctypes
import time

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

WAIT_TIMEOUT = 1          # LA_DEVERR_WAIT_TIMEOUT


@pytest.fixture(scope="module")
def lib():
    from streaming_causal_video_timestep_b200 import _lib, build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return _lib.load()


def test_wait_that_nothing_completes_times_out_and_reports(lib):
    from streaming_causal_video_timestep_b200 import _lib
    word = ctypes.c_int32(-7)
    t0 = time.perf_counter()
    code = lib.la_debug_wait_timeout(50_000_000, 0, ctypes.byref(word))    # 50 ms limit
    elapsed = time.perf_counter() - t0
    assert code == _lib.LA_EDEVICE
    assert word.value == WAIT_TIMEOUT
    assert 0.05 <= elapsed < 5.0


def test_completed_wait_reports_nothing(lib):
    from streaming_causal_video_timestep_b200 import _lib
    word = ctypes.c_int32(-7)
    assert lib.la_debug_wait_timeout(50_000_000, 1, ctypes.byref(word)) == _lib.LA_OK
    assert word.value == 0


def test_context_usable_after_a_timeout(lib):
    from streaming_causal_video_timestep_b200 import _lib, op_euler
    word = ctypes.c_int32(0)
    assert lib.la_debug_wait_timeout(10_000_000, 0, ctypes.byref(word)) == _lib.LA_EDEVICE
    x = torch.ones((256, 64), device="cuda")
    v = torch.full((256, 64), 2.0, device="cuda")
    op_euler(x, v, [-0.25], 256)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(x.cpu().numpy(), np.full((256, 64), 0.5, np.float32))


def test_invalid_limit_is_rejected(lib):
    from streaming_causal_video_timestep_b200 import _lib
    word = ctypes.c_int32(0)
    assert lib.la_debug_wait_timeout(-1, 0, ctypes.byref(word)) == _lib.LA_EINVAL


def test_op_level_wait_timeout_reported_by_op_status_then_cleared(lib):
    """The word the la_op_* kernels (la_op_attention_static included) raise: a
    wait that nothing completes raises it, la_op_status returns LA_EDEVICE once
    and clears it, and an op that then runs is reported clean."""
    from streaming_causal_video_timestep_b200 import _lib, op_euler
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.la_op_status(st) == _lib.LA_OK                  # nothing raised so far in this process
    assert lib.la_debug_op_wait_timeout(20_000_000, st) == _lib.LA_OK
    assert lib.la_op_status(st) == _lib.LA_EDEVICE
    assert lib.la_op_status(st) == _lib.LA_OK                  # cleared by the read
    x = torch.ones((256, 64), device="cuda")
    op_euler(x, torch.full((256, 64), 2.0, device="cuda"), [-0.25], 256)
    assert lib.la_op_status(st) == _lib.LA_OK
    np.testing.assert_array_equal(x.cpu().numpy(), np.full((256, 64), 0.5, np.float32))
    assert lib.la_debug_op_wait_timeout(-1, st) == _lib.LA_EINVAL
