"""FP8 (e4m3) projections on the GPU against the oracle (oracle/fp8.py).

The quantization is an integer decision made in fp32 on both sides, so codes
and scales must match bit for bit.  The GEMM multiplies the 8-bit codes exactly
(a product of two e4m3 values fits fp32) and accumulates in fp32: for any
summation order the error of an output is at most K * 2^-24 times the sum of
the magnitudes of its products, plus the three roundings of the two scale
multiplications and the store, which is the bound the test gates on.
"""
import numpy as np
import pytest

from oracle.fp8 import e4m3_decode, gemm_fp8, quantize_rows
from workloads import bf16_round, random_array

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    from streaming_causal_video_timestep_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")


def _rows(seed, rows, cols):
    x = random_array(seed, (rows, cols)) * np.exp(random_array(seed + 1, (rows, 1)) * 2.0)
    x[rows // 3] = 0.0                                    # an all-zero row: scale 1, codes 0
    return x.astype(np.float32)


@pytest.mark.parametrize("in_dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(300, 1000), (17, 5120), (1, 2)])
def test_quantize_rows_bit_exact(in_dtype, rows, cols):
    from streaming_causal_video_timestep_b200 import op_quantize_e4m3
    x = _rows(3, rows, cols)
    if in_dtype == "bf16":
        x = bf16_round(x).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    if in_dtype == "bf16":
        xt = xt.to(torch.bfloat16)
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    op_quantize_e4m3(xt, codes, scales)
    torch.cuda.synchronize()
    q_ref, s_ref = quantize_rows(x)
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(codes.cpu().numpy(), q_ref)


def _gemm_case(seed, M, N, K):
    a, sa = quantize_rows(_rows(seed, M, K))
    w, sw = quantize_rows((random_array(seed + 7, (N, K)) * 0.02).astype(np.float32))
    return a, sa, w, sw


def _run_gemm(a, sa, w, sw, dtype):
    from streaming_causal_video_timestep_b200 import op_gemm_fp8
    M, N = a.shape[0], w.shape[0]
    out = torch.empty((M, N), dtype=dtype, device="cuda")
    op_gemm_fp8(torch.from_numpy(a).cuda(), torch.from_numpy(sa).cuda(), torch.from_numpy(w).cuda(),
                torch.from_numpy(sw).cuda(), out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(300, 512, 1024), (130, 256, 1040), (4680, 1024, 5120), (33, 96, 16)])
def test_gemm_fp8_within_the_fp32_accumulation_bound(M, N, K):
    a, sa, w, sw = _gemm_case(5, M, N, K)
    got = _run_gemm(a, sa, w, sw, torch.float32)
    ref = gemm_fp8(a, sa, w, sw)
    mag = (np.abs(e4m3_decode(a)) @ np.abs(e4m3_decode(w)).T) * sa.astype(np.float64)[:, None] \
        * sw.astype(np.float64)[None, :]
    bound = (K + 3) * U * mag + 3 * U * np.abs(ref)
    excess = np.abs(got - ref) - bound
    assert np.all(excess <= 0), f"max excess {excess.max():.3e}, max |ref| {np.abs(ref).max():.3e}"


def test_gemm_fp8_bf16_output_is_the_fp32_result_rounded_once():
    a, sa, w, sw = _gemm_case(6, 256, 512, 1024)
    got32 = _run_gemm(a, sa, w, sw, torch.float32)
    got16 = _run_gemm(a, sa, w, sw, torch.bfloat16)
    np.testing.assert_array_equal(got16, bf16_round(got32.astype(np.float32)).astype(np.float64))


def test_quantize_then_gemm_end_to_end_and_report_fp8_error():
    """GPU quantization feeding the GPU GEMM equals the oracle's pipeline within the
    accumulation bound; the error of FP8 against the exact product of the unquantized
    inputs is reported (it is the format's, not the kernel's)."""
    from streaming_causal_video_timestep_b200 import op_gemm_fp8, op_quantize_e4m3
    M, N, K = 512, 1024, 2048
    x = _rows(8, M, K)
    wt = (random_array(9, (N, K)) * 0.02).astype(np.float32)
    dev = lambda t: torch.from_numpy(t).cuda()
    qa, sa = torch.empty((M, K), dtype=torch.uint8, device="cuda"), torch.empty(M, device="cuda")
    qw, sw = torch.empty((N, K), dtype=torch.uint8, device="cuda"), torch.empty(N, device="cuda")
    op_quantize_e4m3(dev(x), qa, sa)
    op_quantize_e4m3(dev(wt), qw, sw)
    out = torch.empty((M, N), device="cuda")
    op_gemm_fp8(qa, sa, qw, sw, out)
    torch.cuda.synchronize()
    a_ref, sa_ref = quantize_rows(x)
    w_ref, sw_ref = quantize_rows(wt)
    np.testing.assert_array_equal(qa.cpu().numpy(), a_ref)
    ref = gemm_fp8(a_ref, sa_ref, w_ref, sw_ref)
    got = out.cpu().numpy().astype(np.float64)
    mag = (np.abs(e4m3_decode(a_ref)) @ np.abs(e4m3_decode(w_ref)).T) * sa_ref[:, None] * sw_ref[None, :]
    assert np.all(np.abs(got - ref) <= (K + 3) * U * mag + 3 * U * np.abs(ref))
    exact = x.astype(np.float64) @ wt.astype(np.float64).T
    rel = np.abs(got - exact).sum() / np.abs(exact).sum()
    print(f"fp8 quantization error vs the unquantized product: sum|d|/sum|ref| = {rel:.3e}")
    assert rel < 0.1
