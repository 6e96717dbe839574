"""Kernel-level parity on the GPU: tcgen05 GEMM epilogues, block attention over
segments (tcgen05 bf16 and SIMT fp32), the Euler update -- each against the
oracle's definition on the same seeded inputs."""
import numpy as np
import pytest

from oracle import block_causal_attention, euler_step
from workloads import DTYPE_BF16, DTYPE_FP32, bf16_round, random_array

from _helpers import assert_close

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from streaming_causal_video_timestep_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")


def _dev(a, dtype):
    tdt = {DTYPE_BF16: torch.bfloat16, DTYPE_FP32: torch.float32}[dtype]
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to("cuda").to(tdt)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


# N = 256 multiples >= 1024 run on CTA pairs (256-row tiles); the others on one CTA
GEMM_SHAPES = [(300, 256, 320), (130, 64, 64), (1000, 1536, 512), (4680 + 37, 192, 64), (17, 512, 1024),
               (17, 1024, 128), (129, 2048, 192), (4680 + 37, 1024, 320), (300, 5120, 64)]


@pytest.mark.parametrize("dtype", [DTYPE_BF16, DTYPE_FP32])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_store_and_resid(dtype, M, N, K):
    from streaming_causal_video_timestep_b200 import op_gemm
    rnd = bf16_round if dtype == DTYPE_BF16 else (lambda a: a.astype(np.float32))
    A = rnd(random_array(M * 7 + N, (M, K)))
    W = rnd(random_array(K * 3 + 1, (N, K), scale=1.0 / np.sqrt(K)))
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    tA, tW = _dev(A, dtype), _dev(W, dtype)
    out = torch.empty((M, N), dtype=tA.dtype, device="cuda")
    op_gemm(tA, tW, "store", out=out)
    torch.cuda.synchronize()
    assert_close(_np(out), ref, dtype, "gemm store")
    # residual: h32 += acc, out = h32 (rounded to dtype)
    h0 = random_array(5, (M, N))
    h32 = torch.from_numpy(h0).cuda()
    out2 = torch.empty((M, N), dtype=tA.dtype, device="cuda")
    op_gemm(tA, tW, "resid", out=out2, h32=h32)
    torch.cuda.synchronize()
    assert_close(_np(h32), h0 + ref, DTYPE_FP32 if dtype == DTYPE_FP32 else dtype, "gemm resid h32")
    if dtype == DTYPE_BF16:
        # the fp32 residual itself carries only fp32 accumulation error
        err = np.abs(_np(h32) - (h0 + ref)).max() / np.abs(h0 + ref).max()
        assert err < 1e-4, err
    assert_close(_np(out2), h0 + ref, dtype, "gemm resid out")


@pytest.mark.parametrize("dtype", [DTYPE_BF16, DTYPE_FP32])
@pytest.mark.parametrize("N", [64, 1024])
def test_gemm_set32_and_euler_epilogues(dtype, N):
    from streaming_causal_video_timestep_b200 import op_gemm
    rnd = bf16_round if dtype == DTYPE_BF16 else (lambda a: a.astype(np.float32))
    M, K, G = 4 * 180, 256, 4
    A = rnd(random_array(1, (M, K)))
    W = rnd(random_array(2, (N, K), scale=0.05))
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    tA, tW = _dev(A, dtype), _dev(W, dtype)
    h32 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    op_gemm(tA, tW, "set32", out=None, h32=h32)
    torch.cuda.synchronize()
    assert_close(_np(h32), ref, DTYPE_FP32 if dtype == DTYPE_FP32 else dtype, "set32")
    x0 = random_array(3, (M, N))
    x = torch.from_numpy(x0).cuda()
    ts = [1.0, 0.75, 0.5, 0.25, 0.0]
    dts = [ts[i + 1] - ts[i] for i in range(G)]
    op_gemm(tA, tW, "euler", h32=x, dt=dts, rows_per_group=M // G)
    torch.cuda.synchronize()
    want = np.concatenate([euler_step(x0[g * 180:(g + 1) * 180], ref[g * 180:(g + 1) * 180], ts[g], ts[g + 1])
                           for g in range(G)])
    assert_close(_np(x), want, DTYPE_FP32 if dtype == DTYPE_FP32 else dtype, "euler epilogue")


def _attn_case(seed, H, d, F, T, nwin, scale=1.0, dtype=DTYPE_BF16, Tq=None):
    rnd = bf16_round if dtype == DTYPE_BF16 else (lambda a: a.astype(np.float32))
    Tq = Tq or T
    q = rnd(random_array(seed, (Tq, H, d), scale))
    sink = (rnd(random_array(seed + 1, (F, H, d), scale)), rnd(random_array(seed + 2, (F, H, d))))
    b = 5
    blocks = {b - nwin + w: (rnd(random_array(seed + 10 + w, (T, H, d), scale)),
                             rnd(random_array(seed + 30 + w, (T, H, d)))) for w in range(nwin + 1)}
    return q, sink, blocks, b


def _run_op_attention(q, sink, blocks, dtype):
    """Returns (output as stored, fp32 output before rounding)."""
    from streaming_causal_video_timestep_b200 import op_attention
    to_planes = lambda a: _dev(np.ascontiguousarray(np.transpose(a, (1, 0, 2))), dtype)
    ks = [to_planes(sink[0])] + [to_planes(blocks[k][0]) for k in sorted(blocks)]
    vs = [to_planes(sink[1])] + [to_planes(blocks[k][1]) for k in sorted(blocks)]
    Tq, H, d = q.shape
    odt = torch.bfloat16 if dtype == DTYPE_BF16 else torch.float32
    out = torch.empty((Tq, H * d), dtype=odt, device="cuda")
    out32 = torch.empty((Tq, H * d), dtype=torch.float32, device="cuda") if dtype == DTYPE_BF16 else None
    op_attention(to_planes(q), ks, vs, out, out32)
    torch.cuda.synchronize()
    return _np(out), (_np(out32) if out32 is not None else _np(out))


@pytest.mark.parametrize("F,T,nwin,scale,Tq", [
    (60, 180, 2, 1.0, None),      # ragged: 180 = 128 + 52, 60 < 128
    (16, 48, 0, 1.0, None),       # no window (block 0)
    (130, 300, 2, 1.0, None),     # several q tiles and key tiles, ragged
    (60, 180, 2, 3.0, None),      # peaked softmax: exercises the lazy O rescale
    (1560, 256, 1, 1.0, 256),     # full-width sink frame
    (60, 180, 2, 300.0, None),    # logits ~1e5: the row max still contributes exactly 1
])
def test_attention_tcgen05_matches_oracle(F, T, nwin, scale, Tq):
    H, d = 2, 128
    q, sink, blocks, b = _attn_case(11, H, d, F, T, nwin, scale, Tq=Tq)
    got, got32 = _run_op_attention(q, sink, blocks, DTYPE_BF16)
    want = block_causal_attention(q, blocks, sink, qblock=b, window=nwin).reshape(q.shape[0], H * d)
    assert_close(got32, want, DTYPE_BF16, "attention fp32 result")
    # the bf16 output (what the output projection consumes) is that result rounded once
    np.testing.assert_array_equal(got, bf16_round(got32.astype(np.float32)))


def test_attention_tcgen05_single_key_passthrough():
    from streaming_causal_video_timestep_b200 import op_attention
    H, d = 3, 128
    q = _dev(random_array(1, (H, 200, d), 5.0), DTYPE_BF16)
    k = _dev(random_array(2, (H, 1, d)), DTYPE_BF16)
    v = _dev(random_array(3, (H, 1, d)), DTYPE_BF16)
    out = torch.empty((200, H * d), dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty((200, H * d), dtype=torch.float32, device="cuda")
    op_attention(q, [k], [v], out, out32)
    torch.cuda.synchronize()
    want = np.broadcast_to(_np(v).transpose(1, 0, 2).reshape(1, H * d), (200, H * d))
    # one visible key: p = 2^0 = 1 exactly, l = 1, so O is V exactly
    np.testing.assert_array_equal(_np(out32), want)


@pytest.mark.parametrize("d", [64, 128])
def test_attention_fp32_matches_oracle(d):
    H, F, T, nwin = 2, 16, 48, 2
    q, sink, blocks, b = _attn_case(21, H, d, F, T, nwin, dtype=DTYPE_FP32)
    got, _ = _run_op_attention(q, sink, blocks, DTYPE_FP32)
    want = block_causal_attention(q, blocks, sink, qblock=b, window=nwin).reshape(T, H * d)
    assert_close(got, want, DTYPE_FP32, "attention fp32")


def test_euler_standalone_matches_oracle():
    from streaming_causal_video_timestep_b200 import op_euler
    rows, C, G = 4 * 4680, 64, 4
    x0 = random_array(7, (rows, C))
    v = random_array(8, (rows, C))
    ts = [1.0, 0.75, 0.5, 0.25, 0.0]
    x = torch.from_numpy(x0).cuda()
    op_euler(x, torch.from_numpy(v).cuda(), [ts[i + 1] - ts[i] for i in range(G)], rows // G)
    torch.cuda.synchronize()
    want = np.concatenate([euler_step(x0[g * 4680:(g + 1) * 4680], v[g * 4680:(g + 1) * 4680], ts[g], ts[g + 1])
                           for g in range(G)])
    assert_close(_np(x), want, DTYPE_FP32, "euler")


@pytest.mark.parametrize("emu", [0, 3, 4])
def test_attention_with_polynomial_exp2_share_matches_oracle(emu, tmp_path):
    """LA_ATTN_EMU=k computes k of every 8 exponential pairs of full key tiles
    with the FMA-pipe polynomial (bf16 default 2, covered by every other
    attention test; 0 is ex2 alone); the setting is read once per process, so
    the case runs in a child process and the parity check runs here."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    out = tmp_path / "attn.npz"
    code = (
        "import sys, numpy as np\n"
        f"sys.path[:0] = [{here!r}, {os.path.dirname(here)!r}]\n"
        "import test_gpu_ops as t\n"
        "from workloads import DTYPE_BF16\n"
        "q, sink, blocks, b = t._attn_case(11, 2, 128, 130, 300, 2)\n"
        "got, got32 = t._run_op_attention(q, sink, blocks, DTYPE_BF16)\n"
        f"np.savez({str(out)!r}, got=got, got32=got32)\n")
    env = dict(os.environ, LA_ATTN_EMU=str(emu))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = np.load(out)
    q, sink, blocks, b = _attn_case(11, 2, 128, 130, 300, 2)
    want = block_causal_attention(q, blocks, sink, qblock=b, window=2).reshape(q.shape[0], 2 * 128)
    assert_close(res["got32"], want, DTYPE_BF16, f"attention fp32 result, polynomial share {emu}/8")
    np.testing.assert_array_equal(res["got"], bf16_round(res["got32"].astype(np.float32)))
