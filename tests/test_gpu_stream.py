"""Stream-level parity on the GPU through the C ABI: every tick's integer state
bit-exact against the oracle's scheduler, and every float intermediate
(q, appended K/V, sink re-rope, attention output, residual after each layer,
velocity, latent) within the stated tolerance, teacher-forced per step."""
import numpy as np
import pytest

from oracle import OracleStream, TickScheduler
from workloads import (BLOCK_DIT, CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP, DTYPE_BF16, block_audio, DTYPE_FP32, SCHED_PIPELINED,
                       SCHED_SEQUENTIAL, SINK_AAS, SINK_FIXED, TINY, StreamConfig, Workload, block_noise, make_weights)

from _helpers import assert_close, errors, make_stream, step_tolerance, to_np
from _percheck import check_sink, check_step, sink_snapshot

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from streaming_causal_video_timestep_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")


SMALL_BF16 = Workload(
    name="small-bf16",
    cfg=StreamConfig(num_layers=2, hidden=256, heads=2, head_dim=128, latent_ch=32, grid_h=6, grid_w=10,
                     window_blocks=2, sink_mode=SINK_AAS, dtype=DTYPE_BF16),
    seed=5, num_blocks=8, w_std=1.5 / 16.0, head_std=0.1)

SMALL_BF16_ID = Workload(
    name="small-bf16-identity",
    cfg=StreamConfig(num_layers=1, hidden=256, heads=2, head_dim=128, latent_ch=256, grid_h=5, grid_w=9,
                     window_blocks=1, sink_mode=SINK_FIXED, timesteps=(0.5, 0.25), dtype=DTYPE_BF16),
    seed=6, num_blocks=4, w_std=1.5 / 16.0)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _run_teacher_forced(wl, check_every_tick=True):
    """Per-op parity of every (block, step) (tests/_percheck.py) plus the
    step-level result: the oracle runs each step in fp64 from the GPU's input
    latent and the GPU's finished block must match it within the stream's
    tolerance."""
    cfg = wl.cfg
    s, W = make_stream(wl, capture=True)
    check_sink(s, cfg, W, W.sink, tag="reference sink")
    orc = OracleStream(cfg, W)
    orc.set_sink(W.sink)
    T, C = cfg.block_tokens, cfg.latent_ch
    x_out = torch.empty((T, C), dtype=torch.float32, device="cuda")
    nb = wl.num_blocks
    S = cfg.num_steps
    per = 8 + 3 * cfg.ring_entries
    report = {}
    drain = S - 1 if cfg.schedule == SCHED_PIPELINED else 0     # the sequential schedule has no pipeline
    has_audio = getattr(cfg, "audio_tokens", 0) > 0
    for k in range(nb + drain):
        xn = block_noise(wl, k) if k < nb else None
        au = block_audio(wl, k) if (k < nb and has_audio) else None
        sink = sink_snapshot(s, cfg)
        fin = s.step(_dev(xn) if xn is not None else None, x_out, audio=_dev(au) if au is not None else None)
        st = s.index_state()
        ran = [(int(st[4 + i * per]), i) for i in range(S) if st[4 + i * per] >= 0]
        if check_every_tick or k >= nb + drain - 1:
            for (b, i) in ran:
                check_step(s, cfg, W, b, i, tag=f"tick {k}", report=report, sink=sink,
                           audio=block_audio(wl, b) if has_audio else None)
        inputs = {(b, i): to_np(s.tap("x_in", 0, i)) for (b, i) in ran}
        got = to_np(x_out).copy() if fin >= 0 else None
        out, fin_o = orc.denoise_step(xn, inputs=inputs, aas_latent=got if fin == 0 else None, audio=au)
        assert fin == fin_o
        np.testing.assert_array_equal(st, orc.index_state())
        if fin >= 0:
            # step-level: the oracle's fp64 chain over the whole step from the GPU's
            # input latent, gated at the stream's tolerance (bf16 / fp32 as stated;
            # e4m3 streams against the oracle's e4m3 definitions, see _helpers)
            report["step-level"] = max(report.get("step-level", (0, 0)),
                                       assert_close(got, out, cfg.dtype, f"finished block {fin} (step-level)",
                                                    tol=step_tolerance(cfg)))
        if fin == 0 and cfg.sink_mode == SINK_AAS:
            check_sink(s, cfg, W, got[:cfg.sink_tokens], tag="AAS sink")
    s.synchronize()
    s.close()
    return report


def test_tiny_fp32_stream_every_tick_matches_oracle():
    _run_teacher_forced(TINY)


@pytest.mark.parametrize("window,nblocks", [(0, 6), (4, 3)])
def test_tiny_fp32_stream_window_edges_match_oracle(window, nblocks):
    """The window's degenerate ends: no prior blocks at all (each block attends to
    the sink and itself), and a stream that ends before its window fills."""
    wl = Workload(f"tiny-w{window}", TINY.cfg.replace(window_blocks=window), TINY.seed, nblocks, TINY.w_std)
    _run_teacher_forced(wl)


def test_small_bf16_stream_window_0_teacher_forced():
    """bf16 with no cache window: ring entries of one block each, sink + self keys."""
    wl = Workload("small-bf16-w0", SMALL_BF16.cfg.replace(window_blocks=0), SMALL_BF16.seed, 6,
                  SMALL_BF16.w_std, SMALL_BF16.head_std)
    _run_teacher_forced(wl)


def test_tiny_fp32_stream_free_running_trajectory():
    """No teacher forcing: the fp32 trajectory itself stays within 1e-5."""
    wl = TINY
    cfg = wl.cfg
    s, W = make_stream(wl)
    orc = OracleStream(cfg, W)
    orc.set_sink(W.sink)
    x_out = torch.empty((cfg.block_tokens, cfg.latent_ch), dtype=torch.float32, device="cuda")
    for k in range(wl.num_blocks + 3):
        xn = block_noise(wl, k) if k < wl.num_blocks else None
        fin = s.step(_dev(xn) if xn is not None else None, x_out)
        out, fin_o = orc.denoise_step(xn)
        assert fin == fin_o
        if fin >= 0:
            assert_close(to_np(x_out), out, DTYPE_FP32, f"block {fin}")
    s.close()


def test_small_bf16_stream_teacher_forced():
    report = _run_teacher_forced(SMALL_BF16)
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


def test_small_bf16_identity_projection_one_slot():
    _run_teacher_forced(SMALL_BF16_ID)


@pytest.mark.parametrize("dtype", [DTYPE_FP32, DTYPE_BF16])
def test_pipelined_equals_sequential_on_gpu_with_fixed_sink(dtype):
    base = TINY if dtype == DTYPE_FP32 else SMALL_BF16
    cfg0 = base.cfg.replace(sink_mode=SINK_FIXED)
    wl = Workload("cmp", cfg0, base.seed, 6, base.w_std, base.head_std)
    W = make_weights(wl)
    outs = {}
    for sched in (SCHED_PIPELINED, SCHED_SEQUENTIAL):
        cfg = cfg0.replace(schedule=sched)
        s, _ = make_stream(wl, W, cfg)
        x_out = torch.empty((cfg.block_tokens, cfg.latent_ch), dtype=torch.float32, device="cuda")
        res = {}
        for k in range(wl.num_blocks + (3 if sched == SCHED_PIPELINED else 0)):
            xn = block_noise(wl, k) if k < wl.num_blocks else None
            fin = s.step(_dev(xn) if xn is not None else None, x_out)
            if fin >= 0:
                res[fin] = to_np(x_out).copy()
        s.close()
        outs[sched] = res
    for b in range(wl.num_blocks):
        # the same kernels on the same rows: identical up to bitwise equality
        np.testing.assert_array_equal(outs[SCHED_PIPELINED][b], outs[SCHED_SEQUENTIAL][b])


def test_index_state_bit_exact_over_long_stream_with_bubbles():
    wl = Workload("idx", TINY.cfg.replace(window_blocks=3), 0, 0, 0.125)
    s, W = make_stream(wl)
    ref = TickScheduler(wl.cfg)
    x = _dev(block_noise(wl, 0))
    x_out = torch.empty_like(x)
    rng = np.random.default_rng(0)
    for k in range(300):
        has_new = bool(rng.random() < 0.85) or k < 5
        fin = s.step(x if has_new else None, x_out)
        run, fin_o = ref.begin_tick(has_new)
        for i, b in run:
            ref.append(i, b)
        ref.end_tick(fin_o)
        assert fin == fin_o
        np.testing.assert_array_equal(s.index_state(), ref.index_state())
    s.synchronize()
    s.close()


def test_state_errors():
    from streaming_causal_video_timestep_b200 import LaError, LaStream
    from _helpers import torch_weights
    wl = TINY
    W = make_weights(wl)
    s = LaStream(wl.cfg, torch_weights(W, wl.cfg))
    x = _dev(block_noise(wl, 0))
    x_out = torch.empty_like(x)
    with pytest.raises(LaError) as e:
        s.step(x, x_out)
    assert e.value.code == -2
    s.set_sink(_dev(W.sink))
    s.step(x, x_out)
    with pytest.raises(LaError) as e:
        s.set_sink(_dev(W.sink))
    assert e.value.code == -2
    with pytest.raises(LaError) as e:
        s.set_slot_input(0, x)
    assert e.value.code == -2
    s.synchronize()
    s.close()
    seq = LaStream(wl.cfg.replace(schedule=SCHED_SEQUENTIAL), torch_weights(W, wl.cfg))
    seq.set_sink(_dev(W.sink))
    with pytest.raises(LaError) as e:
        seq.step(None, x_out)
    assert e.value.code == -1
    seq.close()


@pytest.mark.parametrize("rolling,sink_mode", [(0, SINK_AAS), (0, SINK_FIXED), (1, SINK_FIXED)])
def test_tiny_fp32_ablations_match_oracle(rolling, sink_mode):
    """Ablation schedules on the same kernels: Rolling RoPE off (the sink keeps the
    temporal position of block 0, -3) and / or AAS off (the reference sink for the
    whole stream); integer state bit-exact and every op within 1e-5 every tick."""
    cfg = TINY.cfg.replace(rolling_rope=rolling, sink_mode=sink_mode)
    _run_teacher_forced(Workload(f"tiny-rolling{rolling}-sink{sink_mode}", cfg, TINY.seed, TINY.num_blocks,
                                 TINY.w_std, TINY.head_std))


def test_small_bf16_rolling_rope_off_teacher_forced():
    cfg = SMALL_BF16.cfg.replace(rolling_rope=0)
    _run_teacher_forced(Workload("small-bf16-rolling0", cfg, SMALL_BF16.seed, 6, SMALL_BF16.w_std,
                                 SMALL_BF16.head_std))



def _run_clean_refresh(wl):
    """The clean-cache refresh ablation, free-running: integer state bit-exact and
    the finished block against the oracle every call; returns the worst errors."""
    cfg = wl.cfg
    s, W = make_stream(wl)
    orc = OracleStream(cfg, W)
    orc.set_sink(W.sink)
    x_out = torch.empty((cfg.block_tokens, cfg.latent_ch), dtype=torch.float32, device="cuda")
    worst = (0.0, 0.0)
    for b in range(wl.num_blocks):
        xn = block_noise(wl, b)
        fin = s.step(_dev(xn), x_out)
        out, fin_o = orc.denoise_step(xn)
        assert fin == fin_o == b
        np.testing.assert_array_equal(s.index_state(), orc.index_state())
        if cfg.dtype == DTYPE_FP32:
            assert_close(to_np(x_out), out, DTYPE_FP32, f"clean-refresh block {b}")
        worst = max(worst, errors(to_np(x_out), out))
    s.close()
    return worst


@pytest.mark.parametrize("window", [1, 2])
def test_tiny_fp32_clean_cache_refresh_matches_oracle(window):
    cfg = TINY.cfg.replace(schedule=SCHED_SEQUENTIAL, cache_mode=CACHE_CLEAN_REFRESH, window_blocks=window)
    _run_clean_refresh(Workload(f"tiny-clean-w{window}", cfg, TINY.seed, TINY.num_blocks, TINY.w_std,
                                TINY.head_std))


def test_small_bf16_clean_cache_refresh_integer_state_and_drift():
    cfg = SMALL_BF16.cfg.replace(schedule=SCHED_SEQUENTIAL, cache_mode=CACHE_CLEAN_REFRESH)
    worst = _run_clean_refresh(Workload("small-bf16-clean", cfg, SMALL_BF16.seed, 5, SMALL_BF16.w_std,
                                        SMALL_BF16.head_std))
    print({"free-running drift": (f"{worst[0]:.2e}", f"{worst[1]:.2e}")})


@pytest.mark.parametrize("window,j", [(1, 0), (2, 3), (2, 1)])
def test_tiny_fp32_fixed_noise_cache_matches_oracle(window, j):
    """The fixed-noise cache: every step reads the prior blocks of step j; fp32
    free-running within 1e-5 and the integer state bit-exact every call."""
    cfg = TINY.cfg.replace(schedule=SCHED_SEQUENTIAL, cache_mode=CACHE_FIXED_STEP, cache_step=j,
                           window_blocks=window)
    _run_clean_refresh(Workload(f"tiny-fixed-w{window}-j{j}", cfg, TINY.seed, TINY.num_blocks, TINY.w_std,
                                TINY.head_std))


def test_small_bf16_fixed_noise_cache_teacher_forced():
    cfg = SMALL_BF16.cfg.replace(schedule=SCHED_SEQUENTIAL, cache_mode=CACHE_FIXED_STEP, cache_step=3)
    report = _run_teacher_forced(Workload("small-bf16-fixed", cfg, SMALL_BF16.seed, 5, SMALL_BF16.w_std,
                                          SMALL_BF16.head_std))
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


TINY_DIT = Workload("tiny-dit", TINY.cfg.replace(block_kind=BLOCK_DIT, ffn_dim=160), TINY.seed, TINY.num_blocks,
                    TINY.w_std, TINY.head_std)
SMALL_DIT = Workload("small-bf16-dit", SMALL_BF16.cfg.replace(block_kind=BLOCK_DIT, ffn_dim=640), SMALL_BF16.seed, 6,
                     SMALL_BF16.w_std, SMALL_BF16.head_std)


def test_tiny_fp32_dit_stream_every_tick_matches_oracle():
    """The full DiT block (AdaLN, gated residuals, GELU FFN): every op of every tick
    teacher-forced, and the finished blocks within 1e-5."""
    _run_teacher_forced(TINY_DIT)


def test_tiny_fp32_dit_stream_free_running_and_sequential():
    """Free-running fp32 DiT stream within 1e-5 of the oracle, grouped pipeline and
    sequential schedule (the sequential run also checks the integer state every call)."""
    cfg = TINY_DIT.cfg.replace(schedule=SCHED_SEQUENTIAL)
    _run_clean_refresh(Workload("tiny-dit-seq", cfg, TINY.seed, 5, TINY.w_std, TINY.head_std))
    wl = TINY_DIT
    s, W = make_stream(wl)
    orc = OracleStream(wl.cfg, W)
    orc.set_sink(W.sink)
    x_out = torch.empty((wl.cfg.block_tokens, wl.cfg.latent_ch), dtype=torch.float32, device="cuda")
    for k in range(wl.num_blocks + 3):
        xn = block_noise(wl, k) if k < wl.num_blocks else None
        fin = s.step(_dev(xn) if xn is not None else None, x_out)
        out, fin_o = orc.denoise_step(xn)
        assert fin == fin_o
        if fin >= 0:
            assert_close(to_np(x_out), out, DTYPE_FP32, f"dit block {fin}")
    s.close()


def test_small_bf16_dit_stream_teacher_forced():
    report = _run_teacher_forced(SMALL_DIT)
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


TINY_DIT_AV = Workload("tiny-dit-av", TINY_DIT.cfg.replace(audio_tokens=20, audio_dim=24), TINY.seed, 5,
                       TINY.w_std, TINY.head_std)
SMALL_DIT_AV = Workload("small-bf16-dit-av", SMALL_DIT.cfg.replace(audio_tokens=150, audio_dim=64),
                        SMALL_BF16.seed, 5, SMALL_BF16.w_std, SMALL_BF16.head_std)


def test_tiny_fp32_dit_stream_with_audio_every_tick_matches_oracle():
    """The audio cross-attention: its q, the block's audio K / V, the attention and the
    residual after it per op every tick, and the finished blocks within 1e-5."""
    _run_teacher_forced(TINY_DIT_AV)


def test_small_bf16_dit_stream_with_audio_teacher_forced():
    """150 audio tokens: a full key tile and a ragged one."""
    report = _run_teacher_forced(SMALL_DIT_AV)
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


def test_audio_stream_needs_the_audio():
    from streaming_causal_video_timestep_b200 import LaError
    s, W = make_stream(TINY_DIT_AV)
    x_out = torch.empty((TINY_DIT_AV.cfg.block_tokens, TINY_DIT_AV.cfg.latent_ch), device="cuda")
    with pytest.raises(LaError):
        s.step(_dev(block_noise(TINY_DIT_AV, 0)), x_out)          # no audio
    s.close()


def test_dit_block_rejects_the_e4m3_modes():
    from streaming_causal_video_timestep_b200 import LaError
    with pytest.raises(LaError):
        make_stream(Workload("dit-fp8", SMALL_DIT.cfg.replace(proj_fp8=1), SMALL_DIT.seed, 2, SMALL_DIT.w_std,
                             SMALL_DIT.head_std))


def test_small_bf16_stream_with_e4m3_projections_teacher_forced():
    """e4m3 QKV / output projections: every op of every (block, step) against the
    oracle's quantize-then-multiply definition, integer state bit-exact."""
    cfg = SMALL_BF16.cfg.replace(proj_fp8=1)
    report = _run_teacher_forced(Workload("small-bf16-fp8", cfg, SMALL_BF16.seed, 6, SMALL_BF16.w_std,
                                          SMALL_BF16.head_std))
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


def test_small_bf16_stream_with_e4m3_attention_teacher_forced():
    """e4m3 attention in the denoising passes: per-head scales equal to the oracle's
    rule, the codes of q / ring K, V / re-roped sink K / sink V against the oracle's
    quantization of its own values, the attention from the GPU's codes, integer state
    bit-exact."""
    cfg = SMALL_BF16.cfg.replace(attn_fp8=1)
    report = _run_teacher_forced(Workload("small-bf16-afp8", cfg, SMALL_BF16.seed, 6, SMALL_BF16.w_std,
                                          SMALL_BF16.head_std))
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


def test_small_bf16_stream_with_e4m3_projections_and_attention_teacher_forced():
    cfg = SMALL_BF16.cfg.replace(proj_fp8=1, attn_fp8=1)
    report = _run_teacher_forced(Workload("small-bf16-fp8-all", cfg, SMALL_BF16.seed, 5, SMALL_BF16.w_std,
                                          SMALL_BF16.head_std))
    print({k: (f"{v[0]:.2e}", f"{v[1]:.2e}") for k, v in report.items()})


def test_tiny_fp32_stream_rejects_e4m3_attention():
    from streaming_causal_video_timestep_b200 import LaError
    with pytest.raises(LaError):
        make_stream(Workload("tiny-afp8", TINY.cfg.replace(attn_fp8=1), TINY.seed, 2, TINY.w_std, TINY.head_std))


def test_tiny_fp32_stream_rejects_e4m3_projections():
    from streaming_causal_video_timestep_b200 import LaError
    with pytest.raises(LaError):
        make_stream(Workload("tiny-fp8", TINY.cfg.replace(proj_fp8=1), TINY.seed, 2, TINY.w_std, TINY.head_std))
