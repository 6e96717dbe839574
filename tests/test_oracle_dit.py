"""Pins of the oracle's full DiT block (oracle/dit.py, the BLOCK_DIT stream), CPU only."""
import numpy as np
import pytest
import torch

from oracle import OracleStream
from oracle.dit import ffn, gelu_tanh, modulate
from oracle.norm import rms_norm
from workloads import (BLOCK_ATTN, BLOCK_DIT, SCHED_SEQUENTIAL, SINK_AAS, SINK_FIXED, StreamConfig, Workload,
                       block_noise, make_weights)


def test_gelu_tanh_matches_torch():
    x = np.concatenate([np.linspace(-12, 12, 20001), np.random.default_rng(1).standard_normal(5000) * 3])
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(gelu_tanh(x), ref, rtol=1e-13, atol=1e-15)


def test_modulate_is_the_norm_when_shift_and_scale_vanish_and_affine_otherwise():
    rng = np.random.default_rng(2)
    h = rng.standard_normal((7, 32)) * 5
    z = np.zeros(32)
    np.testing.assert_array_equal(modulate(h, z, z), rms_norm(h))
    sh, sc = rng.standard_normal(32), rng.standard_normal(32)
    np.testing.assert_allclose(modulate(h, sh, sc), rms_norm(h) + rms_norm(h) * sc + sh, rtol=1e-14, atol=1e-14)


def test_ffn_with_identity_weights_is_elementwise_gelu():
    rng = np.random.default_rng(3)
    m = rng.standard_normal((5, 16))
    eye = np.eye(16)
    np.testing.assert_allclose(ffn(m, eye, eye), gelu_tanh(m), rtol=1e-15)
    w1 = rng.standard_normal((24, 16))
    # W2 picks the first 16 of the 24 hidden units
    np.testing.assert_allclose(ffn(m, w1, np.eye(16, 24)), gelu_tanh(m @ w1.T)[:, :16], rtol=1e-14)


def _cfg(**kw):
    base = dict(num_layers=2, hidden=16, heads=2, head_dim=8, latent_ch=16, grid_h=2, grid_w=2, window_blocks=1,
                rope_split=(2, 1, 1), sink_mode=SINK_AAS, dtype=1, block_kind=BLOCK_DIT, ffn_dim=24)
    base.update(kw)
    return StreamConfig(**base)


def _run(cfg, W, wl, nb):
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    outs = {}
    drain = cfg.num_steps - 1 if cfg.schedule == 0 else 0
    for k in range(nb + drain):
        out, fin = s.denoise_step(block_noise(wl, k) if k < nb else None)
        if fin >= 0:
            outs[fin] = out
    return outs


@pytest.mark.parametrize("sink_mode,schedule", [(SINK_AAS, 0), (SINK_FIXED, SCHED_SEQUENTIAL)])
def test_dit_stream_matches_the_scalar_brute_force(sink_mode, schedule):
    cfg = _cfg(sink_mode=sink_mode, schedule=schedule)
    wl = Workload("brute-dit", cfg, 21, 4, 0.25)
    W = make_weights(wl)
    from _brute import BruteStream
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    if schedule == 0:
        want = bs.run_pipelined(noises)
    else:
        want = {}
        for b, nz in enumerate(noises):
            x = [list(map(float, r)) for r in nz]
            for i in range(cfg.num_steps):
                x = bs.step(x, b, i)
            want[b] = x
    got = _run(cfg, W, wl, wl.num_blocks)
    for b in range(wl.num_blocks):
        np.testing.assert_allclose(got[b], np.array(want[b]), rtol=1e-10, atol=1e-10)


def test_dit_with_neutral_adaln_and_no_ffn_is_the_attention_stream():
    """shift = scale = 0, gate1 = 1, gate2 = 0: every layer is the attention sublayer."""
    cfg = _cfg()
    wl = Workload("neutral", cfg, 22, 4, 0.25)
    W = make_weights(wl)
    W.ada[...] = 0.0
    W.ada[:, :, 2] = 1.0
    got = _run(cfg, W, wl, wl.num_blocks)
    ref = _run(cfg.replace(block_kind=BLOCK_ATTN), W, wl, wl.num_blocks)
    for b in range(wl.num_blocks):
        np.testing.assert_allclose(got[b], ref[b], rtol=1e-12, atol=1e-12)


def test_dit_with_closed_gates_leaves_the_residual_unchanged():
    """gate1 = gate2 = 0: h after every layer is the in-projection, so the velocity
    is the head of n(h_in) and one step is x + dt * n(x) (identity in/out maps)."""
    cfg = _cfg(window_blocks=0, sink_mode=SINK_FIXED)
    wl = Workload("closed", cfg, 23, 1, 0.25)
    W = make_weights(wl)
    W.ada[:, :, 2] = 0.0
    W.ada[:, :, 5] = 0.0
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    x = block_noise(wl, 0).astype(np.float64)
    run, _ = s.sched.begin_tick(True)
    got = s.slot_pass(x, 0, 0)
    t = cfg.timesteps
    np.testing.assert_allclose(got, x + (t[1] - t[0]) * rms_norm(x), rtol=1e-13, atol=1e-13)


# -- the audio cross-attention sub-block --------------------------------------------------------
def test_cross_attention_single_audio_token_is_its_value_projected():
    """One audio token: every softmax weight is 1, so the sub-block adds v W_oc^T to every row."""
    from oracle.dit import cross_attention
    rng = np.random.default_rng(31)
    D, H, d, Da = 16, 2, 8, 6
    h = rng.standard_normal((5, D))
    audio = rng.standard_normal((1, Da))
    wqc, wkvc, woc = rng.standard_normal((D, D)), rng.standard_normal((2 * D, Da)), rng.standard_normal((D, D))
    v = (audio @ wkvc.T)[0, D:]
    got = cross_attention(h, audio, wqc, wkvc, woc, H, d)
    np.testing.assert_allclose(got, np.broadcast_to(v @ woc.T, (5, D)), rtol=1e-12, atol=1e-12)


def test_cross_attention_matches_torch_sdpa():
    from oracle.dit import cross_attention
    rng = np.random.default_rng(32)
    D, H, d, Da, T, A = 32, 4, 8, 12, 9, 7
    h = rng.standard_normal((T, D))
    audio = rng.standard_normal((A, Da))
    wqc, wkvc, woc = rng.standard_normal((D, D)), rng.standard_normal((2 * D, Da)), rng.standard_normal((D, D))
    q = (rms_norm(h) @ wqc.T).reshape(T, H, d).transpose(1, 0, 2)
    kv = audio @ wkvc.T
    k = kv[:, :D].reshape(A, H, d).transpose(1, 0, 2)
    v = kv[:, D:].reshape(A, H, d).transpose(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                                         torch.from_numpy(v)).numpy()
    want = o.transpose(1, 0, 2).reshape(T, D) @ woc.T
    np.testing.assert_allclose(cross_attention(h, audio, wqc, wkvc, woc, H, d), want, rtol=1e-11, atol=1e-11)


def test_dit_stream_with_audio_matches_the_scalar_brute_force():
    from workloads import block_audio
    cfg = _cfg(audio_tokens=5, audio_dim=8)
    wl = Workload("brute-dit-audio", cfg, 24, 4, 0.25)
    W = make_weights(wl)
    from _brute import BruteStream
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    audios = [block_audio(wl, b) for b in range(wl.num_blocks)]
    want = bs.run_pipelined(noises, audios)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    got = {}
    for k in range(wl.num_blocks + cfg.num_steps - 1):
        nb = k < wl.num_blocks
        out, fin = s.denoise_step(noises[k] if nb else None, audio=audios[k] if nb else None)
        if fin >= 0:
            got[fin] = out
    for b in range(wl.num_blocks):
        np.testing.assert_allclose(got[b], np.array(want[b]), rtol=1e-10, atol=1e-10)
    # the audio matters
    s2 = OracleStream(cfg.replace(audio_tokens=0), W)
    s2.set_sink(W.sink)
    out0 = [s2.denoise_step(noises[k] if k < 4 else None)[0] for k in range(4 + cfg.num_steps - 1)][-1]
    assert np.abs(out0 - got[3]).max() > 1e-3
