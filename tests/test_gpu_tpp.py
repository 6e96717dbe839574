"""The timestep pipeline across devices, emulated on one GPU: one LA_SCHED_SLOT
stream per denoising step (rank), chained by the same TppRank code that runs the
ranks over torch.distributed (streaming_causal_video_timestep_b200/tpp.py), against
the grouped single-GPU stream.  Each rank's step runs the same kernels on the same
rows as the grouped launch, so the finished blocks are equal bit for bit, with the
Adaptive Attention Sink swapped on every rank by the broadcast from the last rank.
The fp32 chains are also checked against the fp64 oracle's pipelined stream
within 1e-5, free-running."""
import numpy as np
import pytest

from workloads import BLOCK_DIT, DTYPE_BF16, DTYPE_FP32, SCHED_SLOT, SINK_AAS, SINK_FIXED, TINY, StreamConfig, Workload, \
    block_audio, block_noise, make_weights

from oracle import OracleStream

from _helpers import assert_close, make_stream

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from streaming_causal_video_timestep_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")


SMALL = Workload("small-bf16-tpp", StreamConfig(num_layers=2, hidden=256, heads=2, head_dim=128, latent_ch=32,
                                                grid_h=6, grid_w=10, window_blocks=2, sink_mode=SINK_AAS,
                                                dtype=DTYPE_BF16), 5, 7, 1.5 / 16.0, 0.1)
SMALL_DIT_AV = Workload("small-dit-av-tpp", SMALL.cfg.replace(block_kind=BLOCK_DIT, ffn_dim=640, audio_tokens=70,
                                                              audio_dim=64), 5, 6, 1.5 / 16.0, 0.1)


def _grouped(wl, W, audio):
    s, _ = make_stream(wl, W)
    cfg = wl.cfg
    x_out = torch.empty((cfg.block_tokens, cfg.latent_ch), dtype=torch.float32, device="cuda")
    done = {}
    for k in range(wl.num_blocks + cfg.num_steps - 1):
        nb = k < wl.num_blocks
        xn = torch.from_numpy(block_noise(wl, k)).cuda() if nb else None
        au = torch.from_numpy(block_audio(wl, k)).cuda() if (nb and audio) else None
        fin = s.step(xn, x_out, audio=au)
        if fin >= 0:
            done[fin] = x_out.cpu().numpy().copy()
    s.close()
    return done


@pytest.mark.parametrize("wl", [TINY, SMALL, TINY.__class__("tiny-fixed-sink", TINY.cfg.replace(sink_mode=SINK_FIXED),
                                                             TINY.seed, 5, TINY.w_std, TINY.head_std), SMALL_DIT_AV],
                         ids=["tiny-fp32-aas", "small-bf16-aas", "tiny-fp32-fixed", "small-bf16-dit-audio"])
def test_tpp_ranks_on_one_gpu_equal_the_grouped_stream(wl):
    from streaming_causal_video_timestep_b200.tpp import LocalTransport, TppRank, run_local
    cfg = wl.cfg
    W = make_weights(wl)
    audio = getattr(cfg, "audio_tokens", 0) > 0
    want = _grouped(wl, W, audio)
    S = cfg.num_steps
    hub = LocalTransport(S)
    ranks, streams = [], []
    for r in range(S):
        s, _ = make_stream(wl, W, cfg.replace(schedule=SCHED_SLOT, slot_index=r))
        streams.append(s)
        ranks.append(TppRank(s, r, S, hub.endpoint(r), "cuda", S, cfg.sink_tokens, cfg.sink_mode == SINK_AAS,
                             (cfg.audio_tokens, cfg.audio_dim) if audio else None))
    inputs = []
    for k in range(wl.num_blocks + S - 1):
        if k < wl.num_blocks:
            inputs.append((torch.from_numpy(block_noise(wl, k)).cuda(),
                           torch.from_numpy(block_audio(wl, k)).cuda() if audio else None))
        else:
            inputs.append(None)
    got = run_local(ranks, inputs)
    for r in ranks:
        r.close()
    for s in streams:
        s.synchronize()
        s.close()
    assert sorted(got) == list(range(wl.num_blocks))
    for b in range(wl.num_blocks):
        np.testing.assert_array_equal(got[b].cpu().numpy(), want[b])
    if cfg.dtype == DTYPE_FP32:
        # and against the fp64 oracle's single-process pipelined stream, free-running,
        # within the fp32 tolerance (no teacher forcing: the whole trajectory)
        orc = OracleStream(cfg, W)
        orc.set_sink(W.sink)
        ref = {}
        for k in range(wl.num_blocks + S - 1):
            out, fin = orc.denoise_step(block_noise(wl, k) if k < wl.num_blocks else None)
            if fin >= 0:
                ref[fin] = out
        assert sorted(ref) == list(range(wl.num_blocks))
        for b in range(wl.num_blocks):
            assert_close(got[b].cpu().numpy(), ref[b], DTYPE_FP32, f"TPP rank chain, block {b}")


def test_slot_stream_rejects_other_cache_modes_and_a_second_sink_swap():
    from streaming_causal_video_timestep_b200 import LaError
    from workloads import CACHE_CLEAN_REFRESH
    with pytest.raises(LaError):
        make_stream(TINY, None, TINY.cfg.replace(schedule=SCHED_SLOT, slot_index=1, cache_mode=CACHE_CLEAN_REFRESH))
    s, W = make_stream(TINY, None, TINY.cfg.replace(schedule=SCHED_SLOT, slot_index=2))
    sink = torch.from_numpy(W.sink).cuda()
    s.replace_sink(sink)
    with pytest.raises(LaError):
        s.replace_sink(sink)
    s.close()
    g, _ = make_stream(TINY)
    with pytest.raises(LaError):
        g.replace_sink(sink)                 # the grouped stream swaps its sink itself
    g.close()
