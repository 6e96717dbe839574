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

from oracle import block_causal_attention
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


# ---- FP8 attention ---------------------------------------------------------------------
# The oracle (oracle.fp8.attention_fp8) fixes the e4m3 rounding of P against the final
# whole-number row max; the kernel forms P against a running whole-number max and
# rescales O by exact powers of two, so its codes are the same wherever they are normal
# e4m3 values.  The remaining differences are fp32 rounding (scores, ex2, sums) and the
# rare P codes that fp32 rounding moves across an e4m3 rounding boundary.  The gate is
# the stated bf16 tolerance on the fp32 result.
from _helpers import assert_close, errors  # noqa: E402
from oracle.fp8 import attention_fp8  # noqa: E402
from workloads import DTYPE_BF16  # noqa: E402


def _codes(seed, shape, sigma=1.0):
    """e4m3 codes of N(0, sigma^2) values clipped to +-448 (torch's float8_e4m3fn
    conversion, which does not saturate)."""
    x = torch.from_numpy(np.clip(random_array(seed, shape, sigma), -448.0, 448.0))
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _fp8_attn_case(seed, H, Tq, seg_lens, sigma_q=1.0):
    q = _codes(seed, (Tq, H, 128), sigma_q)
    ks = [_codes(seed + 10 + i, (n, H, 128)) for i, n in enumerate(seg_lens)]
    vs = [_codes(seed + 40 + i, (n, H, 128)) for i, n in enumerate(seg_lens)]
    rng = np.random.default_rng(seed + 99)
    sq = np.float32(2.0) ** rng.integers(-2, 2, H).astype(np.float32)
    sk = (rng.uniform(0.3, 1.0, H)).astype(np.float32)
    sv = (rng.uniform(0.5, 2.0, H)).astype(np.float32)
    return q, ks, vs, sq, sk, sv


def _run_fp8_attention(q, ks, vs, sq, sk, sv):
    from streaming_causal_video_timestep_b200 import op_attention_fp8
    planes = lambda a: torch.from_numpy(np.ascontiguousarray(np.transpose(a, (1, 0, 2)))).cuda()
    Tq, H, d = q.shape
    out = torch.empty((Tq, H * d), dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty((Tq, H * d), dtype=torch.float32, device="cuda")
    vec = lambda a: torch.from_numpy(np.asarray(a, np.float32)).cuda()
    op_attention_fp8(planes(q), [planes(k) for k in ks], [planes(v) for v in vs], vec(sq), vec(sk), vec(sv),
                     out, out32)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), out32.cpu().numpy()


@pytest.mark.parametrize("Tq,seg_lens,sigma_q", [
    (300, [60, 180, 180, 130], 1.0),     # ragged queries (2 + 1 tiles) and ragged key segments
    (128, [1], 1.0),                     # one key
    (200, [128, 256], 1.0),              # whole key tiles only
    (180, [60, 180, 180], 4.0),          # peaked softmax: the running max is raised
    (180, [60, 180, 180], 60.0),         # huge scores (codes up to 448)
])
def test_attention_fp8_matches_oracle(Tq, seg_lens, sigma_q):
    H = 2
    q, ks, vs, sq, sk, sv = _fp8_attn_case(31, H, Tq, seg_lens, sigma_q)
    got, got32 = _run_fp8_attention(q, ks, vs, sq, sk, sv)
    want = attention_fp8(q, np.concatenate(ks), np.concatenate(vs), sq, sk, sv).reshape(Tq, H * 128)
    max_rel, mean_rel = assert_close(got32, want, DTYPE_BF16, "fp8 attention fp32 result")
    print(f"fp8 attention vs oracle: max {max_rel:.2e}, mean {mean_rel:.2e}")
    np.testing.assert_array_equal(got, bf16_round(got32))


def test_attention_fp8_stream_shape_sampled_rows():
    """The 14B-like slot: 4680 queries against sink 1560 + window 2 x 4680 + block 4680
    keys, two heads; the oracle computes a sample of query rows (each row is independent
    given every key) including both ends of every query tile pair."""
    H, Tq = 2, 4680
    seg_lens = [1560, 4680, 4680, 4680]
    q, ks, vs, sq, sk, sv = _fp8_attn_case(41, H, Tq, seg_lens)
    got, got32 = _run_fp8_attention(q, ks, vs, sq, sk, sv)
    rows = np.unique(np.concatenate([np.arange(0, Tq, 37), [127, 128, 255, 256, Tq - 1]]))
    want = attention_fp8(q[rows], np.concatenate(ks), np.concatenate(vs), sq, sk, sv).reshape(len(rows), H * 128)
    max_rel, mean_rel = assert_close(got32[rows], want, DTYPE_BF16, "fp8 attention, sampled rows")
    print(f"fp8 attention (stream shape) vs oracle: max {max_rel:.2e}, mean {mean_rel:.2e}")


def test_attention_fp8_whole_number_scores_give_exact_softmax_attention():
    """Scores that are whole numbers in the log2 domain make every P a power of two,
    which e4m3 holds exactly; the result is then plain softmax attention of the
    dequantized operands (oracle.block_causal_attention)."""
    H, Tq, N, d = 2, 256, 300, 128
    rng = np.random.default_rng(5)
    q = np.zeros((Tq, H, d), np.float32)
    k = np.zeros((N, H, d), np.float32)
    q[:, :, 0] = rng.choice([1.0, 2.0], (Tq, H))
    k[:, :, 0] = rng.integers(-4, 3, (N, H))
    v = random_array(6, (N, H, d))
    f8 = lambda a: torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    qc, kc, vc = f8(q), f8(k), f8(v)
    sq = np.float32([1.0, 1.0])
    sk = np.float32([np.sqrt(d) / np.log2(np.e)] * H)
    sv = np.float32([1.0, 0.5])
    _, got32 = _run_fp8_attention(qc, [kc[:100], kc[100:]], [vc[:100], vc[100:]], sq, sk, sv)
    deq = lambda c, s: e4m3_decode(c) * s[None, :, None].astype(np.float64)
    want = block_causal_attention(deq(qc, sq), {0: (deq(kc, sk), deq(vc, sv))}, None, qblock=0,
                                  window=0).reshape(Tq, H * d)
    max_rel, mean_rel = errors(got32, want)
    assert max_rel <= 1e-5 and mean_rel <= 1e-5, (max_rel, mean_rel)
