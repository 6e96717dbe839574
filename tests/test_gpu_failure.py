"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up after its limit, raises the device error word and returns;
the host reads LA_EDEVICE and the context stays usable."""
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
