"""Pins of the fp64 oracle against things other than itself (CPU only).

Brute force on tiny inputs, a library special case (SDPA), closed forms,
invariants, and values the Live Avatar pages print (tests/golden).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import OracleStream, TickScheduler, block_causal_attention, euler_step, rms_norm, rope_rotate
from oracle.rope import axis_frequencies, block_positions, sink_positions, sink_temporal_position
from workloads import (CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP, CACHE_TIMESTEP, SCHED_PIPELINED, SCHED_SEQUENTIAL,
                       SINK_AAS, SINK_FIXED, TINY, StreamConfig, Workload, block_noise, make_weights, random_array)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)


def _tiny_blocks(rng, nblocks, T, H, d):
    return {b: (rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d))) for b in nblocks}


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def test_attention_matches_per_query_brute_force():
    rng = np.random.default_rng(1)
    T, F, H, d, window = 12, 4, 2, 4, 2
    qblock = 5
    # blocks 2 (evicted: outside the window), 3, 4 (window), 5 (self), 6 (future)
    blocks = _tiny_blocks(rng, [2, 3, 4, 5, 6], T, H, d)
    sink = (rng.standard_normal((F, H, d)), rng.standard_normal((F, H, d)))
    q = rng.standard_normal((T, H, d))
    got = block_causal_attention(q, blocks, sink, qblock=qblock, window=window)
    for t in range(T):
        for h in range(H):
            keys = [(sink[0][n, h], sink[1][n, h]) for n in range(F)]
            for b, (k, v) in blocks.items():
                if qblock - window <= b <= qblock:
                    keys += [(k[n, h], v[n, h]) for n in range(T)]
            logits = [sum(q[t, h, e] * kk[e] for e in range(d)) / math.sqrt(d) for kk, _ in keys]
            mx = max(logits)
            w = [math.exp(z - mx) for z in logits]
            tot = sum(w)
            want = [sum(wi / tot * vv[e] for wi, (_, vv) in zip(w, keys)) for e in range(d)]
            np.testing.assert_allclose(got[t, h], want, rtol=1e-12, atol=1e-13)


def test_attention_matches_sdpa_on_visible_segments():
    rng = np.random.default_rng(2)
    T, F, H, d, window = 48, 16, 3, 8, 2
    qblock = 7
    blocks = _tiny_blocks(rng, [3, 4, 5, 6, 7], T, H, d)
    sink = (rng.standard_normal((F, H, d)), rng.standard_normal((F, H, d)))
    q = rng.standard_normal((T, H, d))
    got = block_causal_attention(q, blocks, sink, qblock=qblock, window=window)
    seg_k = [sink[0]] + [blocks[b][0] for b in (5, 6, 7)]
    seg_v = [sink[1]] + [blocks[b][1] for b in (5, 6, 7)]
    K = torch.from_numpy(np.concatenate(seg_k)).permute(1, 0, 2)
    V = torch.from_numpy(np.concatenate(seg_v)).permute(1, 0, 2)
    Q = torch.from_numpy(q).permute(1, 0, 2)
    want = torch.nn.functional.scaled_dot_product_attention(Q, K, V).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_softmax_rows_sum_to_one_and_masked_keys_get_zero():
    rng = np.random.default_rng(3)
    T, F, H, d = 12, 4, 2, 4
    blocks = _tiny_blocks(rng, [0, 1, 2, 3], T, H, d)
    sink = (rng.standard_normal((F, H, d)), rng.standard_normal((F, H, d)))
    q = rng.standard_normal((T, H, d)) * 3
    _, p, mask = block_causal_attention(q, blocks, sink, qblock=3, window=1, return_probs=True)
    np.testing.assert_allclose(p.sum(axis=2), 1.0, rtol=0, atol=1e-14)
    assert np.all(p[:, :, ~mask[0]] == 0.0)
    # visible keys: 4 sink + block 2 + block 3
    assert mask[0].sum() == F + 2 * T


def test_single_visible_key_passes_its_value_through():
    rng = np.random.default_rng(4)
    H, d = 2, 8
    sink = (rng.standard_normal((1, H, d)), rng.standard_normal((1, H, d)))
    q = rng.standard_normal((5, H, d)) * 10
    got = block_causal_attention(q, {}, sink, qblock=0, window=2)
    np.testing.assert_array_equal(got, np.broadcast_to(sink[1], got.shape))


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
PAIRS = (22, 21, 21)


def _complex_rope(x, t, r, c, pairs, theta):
    """Independent formulation: pairs as complex numbers times exp(i * angle)."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    pt, ph, pw = pairs
    ang = np.concatenate([t * theta ** (-np.arange(pt) / pt), r * theta ** (-np.arange(ph) / ph),
                          c * theta ** (-np.arange(pw) / pw)])
    z = z * np.exp(1j * ang)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 3, 128))
    t = np.array([0, 1, 5, 29999, -3, 7])
    r = np.array([0, 3, 29, 1, 0, 12])
    c = np.array([0, 51, 2, 7, 0, 40])
    got = rope_rotate(x, t, r, c, PAIRS, 10000.0)
    for n in range(6):
        want = _complex_rope(x[n], t[n], r[n], c[n], PAIRS, 10000.0)
        np.testing.assert_allclose(got[n], want, rtol=1e-12, atol=1e-12)


def test_rope_preserves_norm_and_identity_at_origin():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((10, 2, 64))
    pos = rng.integers(-50, 5000, size=(3, 10))
    y = rope_rotate(x, *pos, (12, 10, 10), 10000.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    z = rope_rotate(x, np.zeros(10), np.zeros(10), np.zeros(10), (12, 10, 10), 10000.0)
    np.testing.assert_allclose(z, x, rtol=0, atol=0)


def test_rope_relative_position_identity():
    """R(a)^T R(b) = R(b - a): q(P) . k(p) depends only on P - p, per axis."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 128))
    k = rng.standard_normal((1, 128))
    P = np.array([[40], [3], [9]])
    p = np.array([[37], [5], [1]])
    base = (rope_rotate(q, *P, PAIRS, 1e4) * rope_rotate(k, *p, PAIRS, 1e4)).sum()
    for shift in ([100, 0, 0], [0, 7, -2], [29996, 11, 13]):
        s = np.array(shift)[:, None]
        moved = (rope_rotate(q, *(P + s), PAIRS, 1e4) * rope_rotate(k, *(p + s), PAIRS, 1e4)).sum()
        assert abs(moved - base) < 1e-9 * max(1.0, abs(base))
    # and equals q . R(p - P) k
    rel = (q * rope_rotate(k, *(p - P), PAIRS, 1e4)).sum()
    assert abs(rel - base) < 1e-10 * max(1.0, abs(base))


def test_axis_frequencies_follow_theta_power_rule():
    wt, wh, ww = axis_frequencies((22, 21, 21), 10000.0)
    assert wt[0] == 1.0 and wh[0] == 1.0 and ww[0] == 1.0
    np.testing.assert_allclose(wt[11] ** 2, 10000.0 ** (-1.0), rtol=1e-14)   # theta^(-11/22)
    np.testing.assert_allclose(wh[7] ** 3, 10000.0 ** (-1.0), rtol=1e-14)    # theta^(-7/21)


def test_block_positions_frame_major_then_row_then_column():
    cfg = TINY.cfg.replace(grid_h=2, grid_w=3)
    t, r, c = block_positions(cfg, 4)
    assert list(t) == [12] * 6 + [13] * 6 + [14] * 6
    assert list(r[:6]) == [0, 0, 0, 1, 1, 1]
    assert list(c[:6]) == [0, 1, 2, 0, 1, 2]


# ---------------------------------------------------------------------------
# Rolling RoPE
# ---------------------------------------------------------------------------
def test_rolling_rope_keeps_sink_offset_constant_to_10000_blocks():
    cfg = TINY.cfg
    for b in range(0, 10001):
        assert sink_temporal_position(cfg, b) - cfg.frames_per_block * b == -3
    fixed = cfg.replace(rolling_rope=0)
    assert sink_temporal_position(fixed, 10000) == -3


def test_rolling_rope_sink_logits_identical_at_block_1_and_10000():
    cfg = TINY.cfg.replace(head_dim=128, hidden=128, rope_split=PAIRS)
    rng = np.random.default_rng(8)
    qb = rng.standard_normal((cfg.block_tokens, 1, 128))
    ks = rng.standard_normal((cfg.sink_tokens, 1, 128))

    def logits(b):
        q = rope_rotate(qb, *block_positions(cfg, b), cfg.pairs, cfg.rope_theta)
        k = rope_rotate(ks, *sink_positions(cfg, sink_temporal_position(cfg, b)), cfg.pairs,
                        cfg.rope_theta)
        return q[:, 0] @ k[:, 0].T

    np.testing.assert_allclose(logits(10000), logits(1), rtol=1e-9, atol=1e-9)
    # without rolling the sink's distance grows and the logits differ
    cfg_fixed = cfg.replace(rolling_rope=0)
    q = rope_rotate(qb, *block_positions(cfg_fixed, 10000), cfg.pairs, cfg.rope_theta)
    k = rope_rotate(ks, *sink_positions(cfg_fixed, -3), cfg.pairs, cfg.rope_theta)
    assert np.abs(q[:, 0] @ k[:, 0].T - logits(1)).max() > 1e-3


# ---------------------------------------------------------------------------
# flow matching
# ---------------------------------------------------------------------------
def test_constant_velocity_reproduces_straight_path_exactly():
    rng = np.random.default_rng(9)
    x0 = rng.standard_normal((48, 64))
    x1 = rng.standard_normal((48, 64))
    ts = TINY.cfg.timesteps
    x = x1.copy()                 # t = 1
    for i in range(len(ts) - 1):
        x = euler_step(x, x1 - x0, ts[i], ts[i + 1])
        np.testing.assert_allclose(x, ts[i + 1] * x1 + (1 - ts[i + 1]) * x0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(x, x0, atol=1e-14)


# ---------------------------------------------------------------------------
# schedule, timestep forcing, AAS
# ---------------------------------------------------------------------------
def test_scheduler_closed_form_uninterrupted_stream():
    cfg = TINY.cfg
    sch = TickScheduler(cfg)
    S, E, nw = cfg.num_steps, cfg.ring_entries, cfg.window_blocks
    nb = 40
    for k in range(nb + S - 1):
        run, fin = sch.begin_tick(k < nb)
        assert run == [(i, k - i) for i in range(S) if 0 <= k - i < nb]
        assert fin == (k - S + 1 if k - S + 1 >= 0 else -1)
        for i, b in run:
            rec = sch.append(i, b)
            assert rec[0] == b and rec[1] == b % E
            assert rec[2] == (b - E if b >= E else -1)
            assert rec[3] == 3 * b - 3 and rec[4] == 3 * b
            resident = list(range(max(0, b - nw), b + 1))
            assert rec[7] == len(resident) and rec[8:8 + len(resident)] == resident
            assert sch.window_blocks(i, b) == resident[:-1]
        sch.end_tick(fin)
    assert sch.blocks_out == nb


def test_timestep_forcing_every_cache_entry_holds_its_own_step():
    wl = TINY
    W = make_weights(wl)
    s = OracleStream(wl.cfg, W)
    s.set_sink(W.sink)
    for k in range(wl.num_blocks + 3):
        s.denoise_step(block_noise(wl, k) if k < wl.num_blocks else None)
        for (l, i, b), (_, _, tag) in s.cache.items():
            assert tag == (b, i)
        for i in range(wl.cfg.num_steps):
            for (blk, step) in s.sched.tags[i]:
                assert blk == -1 or step == i


def test_each_block_takes_exactly_nfe_forward_passes_and_sink_replaced_once():
    facts = _facts()
    wl = TINY
    W = make_weights(wl)
    s = OracleStream(wl.cfg, W, trace=True)
    s.set_sink(W.sink)
    gens = []
    out0 = None
    for k in range(wl.num_blocks + 3):
        out, fin = s.denoise_step(block_noise(wl, k) if k < wl.num_blocks else None)
        if fin == 0:
            out0 = out
        gens.append(s.sched.sink_generation)
    passes = {}
    for key in s.trace:
        if isinstance(key[0], int):
            passes[key[0]] = passes.get(key[0], 0) + 1
    assert set(passes.values()) == {facts["nfe_per_block_no_refresh"]["value"]}
    assert wl.cfg.frames_per_block == facts["frames_per_block"]["value"]
    assert wl.cfg.num_steps == facts["pipeline_workers"]["value"]
    # sink replaced once, right after block 0 finished (tick 3), never again
    assert gens == [0, 0, 0, 1, 1, 1, 1, 1, 1]
    assert gens.count(0) == 3 and sorted(set(gens)) == [0, facts["sink_replacements"]["value"]]
    np.testing.assert_array_equal(s.sink_latent, out0[: wl.cfg.sink_tokens])


def test_pipelined_order_equals_sequential_order_with_fixed_sink():
    wl = Workload("t", TINY.cfg.replace(sink_mode=SINK_FIXED, num_layers=2), 3, 7, 0.125)
    W = make_weights(wl)
    outs = {}
    for sched in (SCHED_PIPELINED, SCHED_SEQUENTIAL):
        cfg = wl.cfg.replace(schedule=sched)
        s = OracleStream(cfg, W)
        s.set_sink(W.sink)
        res = {}
        n_calls = wl.num_blocks + (3 if sched == SCHED_PIPELINED else 0)
        for k in range(n_calls):
            out, fin = s.denoise_step(block_noise(wl, k) if k < wl.num_blocks else None)
            if fin >= 0:
                res[fin] = out
        outs[sched] = res
    assert sorted(outs[0]) == list(range(wl.num_blocks))
    for b in range(wl.num_blocks):
        np.testing.assert_array_equal(outs[SCHED_PIPELINED][b], outs[SCHED_SEQUENTIAL][b])


def test_pipelined_differs_from_sequential_with_aas():
    """The AAS sink reaches blocks 1-3 only for their later steps in pipelined order."""
    wl = Workload("t", TINY.cfg.replace(sink_mode=SINK_AAS), 3, 5, 0.125)
    W = make_weights(wl)
    res = {}
    for sched in (SCHED_PIPELINED, SCHED_SEQUENTIAL):
        s = OracleStream(wl.cfg.replace(schedule=sched), W)
        s.set_sink(W.sink)
        got = {}
        for k in range(wl.num_blocks + (3 if sched == SCHED_PIPELINED else 0)):
            out, fin = s.denoise_step(block_noise(wl, k) if k < wl.num_blocks else None)
            if fin >= 0:
                got[fin] = out
        res[sched] = got
    np.testing.assert_array_equal(res[0][0], res[1][0])
    assert np.abs(res[0][1] - res[1][1]).max() > 1e-6


# ---------------------------------------------------------------------------
# closed forms of the whole step with special weights
# ---------------------------------------------------------------------------
def _special_weights(cfg, q_scale=0.0, k_scale=0.0, out_scale=1.0, sink=None):
    D = cfg.hidden
    wqkv = np.zeros((3 * D, D), np.float32)
    wqkv[0:D] = np.eye(D) * q_scale
    wqkv[D:2 * D] = np.eye(D) * k_scale
    wqkv[2 * D:3 * D] = np.eye(D)
    wout = np.eye(D, dtype=np.float32) * out_scale

    class W:
        pass
    w = W()
    w.w_qkv = [wqkv] * cfg.num_layers
    w.w_out = [wout] * cfg.num_layers
    w.w_in = None
    w.w_head = None
    w.sink = sink
    return w


def test_uniform_attention_closed_form_counts_the_visible_tokens():
    """With W_q = W_k = 0, W_v = W_out = I and identity in/head projections the
    layer adds the mean of the visible tokens' normalised inputs, so one step
    gives x' = x + dt n(x + mean(n(sink), n(window inputs at this step), n(x)))
    with n the per-token RMS normalisation."""
    cfg = TINY.cfg.replace(sink_mode=SINK_FIXED, window_blocks=2)
    rng = np.random.default_rng(10)
    sink = rng.standard_normal((cfg.sink_tokens, cfg.hidden)).astype(np.float32)
    W = _special_weights(cfg, sink=sink)
    s = OracleStream(cfg, W, trace=True)
    s.set_sink(sink)
    nrm = lambda a: a / np.sqrt((a.astype(np.float64) ** 2).mean(axis=-1, keepdims=True) + 1e-6)
    # the sink's stored V is its normalised latent
    np.testing.assert_allclose(s.sink_v[0].reshape(cfg.sink_tokens, -1), nrm(sink), rtol=1e-12, atol=1e-12)
    nb = 6
    for k in range(nb + 3):
        s.denoise_step(block_noise(Workload("n", cfg, 5, nb, 0.1), k) if k < nb else None)
    for (b, i), tr in [(key, v) for key, v in s.trace.items() if isinstance(key[0], int)]:
        x = tr["x_in"]
        toks = [nrm(sink)] + [nrm(s.trace[(bb, i)]["x_in"]) for bb in range(max(0, b - 2), b)] + [nrm(x)]
        mean = np.concatenate(toks).mean(axis=0)
        dt = cfg.timesteps[i + 1] - cfg.timesteps[i]
        np.testing.assert_allclose(tr["x_out"], x + dt * nrm(x + mean[None, :]), rtol=1e-12, atol=1e-12)


def test_rms_norm_matches_torch_and_is_scale_free():
    rng = np.random.default_rng(12)
    h = rng.standard_normal((7, 64)) * rng.uniform(0.01, 1e4, size=(7, 1))
    want = torch.nn.functional.rms_norm(torch.from_numpy(h), (64,), eps=1e-6).numpy()
    np.testing.assert_allclose(rms_norm(h), want, rtol=1e-12, atol=1e-12)
    big = rms_norm(h * 1e3)
    np.testing.assert_allclose(np.sqrt((big ** 2).mean(axis=-1)), 1.0, rtol=1e-9)
    np.testing.assert_allclose(big, rms_norm(h), rtol=1e-6)


def test_oracle_stream_matches_scalar_brute_force_stream():
    from _brute import BruteStream
    cfg = StreamConfig(num_layers=2, hidden=16, heads=2, head_dim=8, latent_ch=16, grid_h=2,
                       grid_w=2, window_blocks=1, rope_split=(2, 1, 1), sink_mode=SINK_AAS,
                       dtype=1)
    wl = Workload("brute", cfg, 11, 5, 0.25)
    W = make_weights(wl)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    want = bs.run_pipelined(noises)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    for k in range(wl.num_blocks + 3):
        out, fin = s.denoise_step(noises[k] if k < wl.num_blocks else None)
        if fin >= 0:
            np.testing.assert_allclose(out, np.array(want[fin]), rtol=1e-11, atol=1e-11)


def test_oracle_stream_matches_brute_force_with_projections_and_no_rolling():
    from _brute import BruteStream
    cfg = StreamConfig(num_layers=1, hidden=16, heads=1, head_dim=16, latent_ch=4, grid_h=1,
                       grid_w=3, window_blocks=2, rope_split=(4, 2, 2), sink_mode=SINK_FIXED,
                       rolling_rope=0, timesteps=(1.0, 0.6, 0.2, 0.0), dtype=1)
    wl = Workload("brute2", cfg, 12, 6, 0.3, head_std=0.3)
    W = make_weights(wl)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    want = bs.run_pipelined(noises)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    for k in range(wl.num_blocks + cfg.num_steps - 1):
        out, fin = s.denoise_step(noises[k] if k < wl.num_blocks else None)
        if fin >= 0:
            np.testing.assert_allclose(out, np.array(want[fin]), rtol=1e-11, atol=1e-11)


# -- the clean-cache refresh ablation (NFE num_steps + 1) ---------------------------------------
def _clean_cfg(**kw):
    base = dict(num_layers=2, hidden=16, heads=2, head_dim=8, latent_ch=16, grid_h=2, grid_w=2, window_blocks=1,
                rope_split=(2, 1, 1), sink_mode=SINK_AAS, dtype=1, schedule=SCHED_SEQUENTIAL,
                cache_mode=CACHE_CLEAN_REFRESH)
    base.update(kw)
    return StreamConfig(**base)


@pytest.mark.parametrize("window,sink_mode,rolling", [(1, SINK_AAS, 1), (2, SINK_FIXED, 0)])
def test_clean_refresh_oracle_matches_scalar_brute_force(window, sink_mode, rolling):
    cfg = _clean_cfg(window_blocks=window, sink_mode=sink_mode, rolling_rope=rolling)
    wl = Workload("brute-clean", cfg, 13, 5, 0.25)
    W = make_weights(wl)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    from _brute import BruteStream
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    want = bs.run_sequential_clean(noises)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    for b in range(wl.num_blocks):
        out, fin = s.denoise_step(noises[b])
        assert fin == b
        np.testing.assert_allclose(out, np.array(want[b]), rtol=1e-11, atol=1e-11)


def test_clean_refresh_equals_timestep_forcing_without_a_window():
    """Window 0: no step reads a cache entry of another block, so the two cache
    modes compute the same latents (the refresh leaves x unchanged)."""
    outs = {}
    for mode in (CACHE_TIMESTEP, CACHE_CLEAN_REFRESH):
        cfg = _clean_cfg(window_blocks=0, cache_mode=mode)
        wl = Workload("w0", cfg, 14, 4, 0.25)
        W = make_weights(wl)
        s = OracleStream(cfg, W)
        s.set_sink(W.sink)
        outs[mode] = [s.denoise_step(block_noise(wl, b))[0] for b in range(wl.num_blocks)]
    for a, b in zip(outs[CACHE_TIMESTEP], outs[CACHE_CLEAN_REFRESH]):
        np.testing.assert_array_equal(a, b)


def test_clean_refresh_ring_tags_closed_form():
    """One shared ring: after block b, entry b mod (window+1) holds (b, S) (the
    refresh), the resident blocks are b-window .. b, and every step's record
    shows that ring."""
    cfg = _clean_cfg(window_blocks=2)
    wl = Workload("tags", cfg, 15, 6, 0.25)
    W = make_weights(wl)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    S, E = cfg.num_steps, cfg.ring_entries
    _, per, _ = __import__("oracle").index_state_layout(cfg)
    for b in range(wl.num_blocks):
        s.denoise_step(block_noise(wl, b))
        st = s.index_state()
        tags = {(b2 % E): (b2, S) for b2 in range(max(0, b - 2), b + 1)}
        for i in range(S):
            rec = st[4 + i * per: 4 + (i + 1) * per]
            assert rec[0] == b and rec[1] == b % E and rec[6] == i
            assert list(rec[8:8 + E]) == list(range(max(0, b - 2), b + 1)) + [-1] * (E - min(b + 1, E))
            got = {e: (rec[8 + E + 2 * e], rec[8 + E + 2 * e + 1]) for e in range(E) if rec[8 + E + 2 * e] >= 0}
            assert got == tags


def test_clean_refresh_needs_the_sequential_schedule():
    with pytest.raises(ValueError):
        TickScheduler(_clean_cfg(schedule=SCHED_PIPELINED))


# -- the fixed-noise cache (every step reads the prior blocks of one step) ------------------------
@pytest.mark.parametrize("window,j,sink_mode", [(1, 0, SINK_AAS), (2, 3, SINK_AAS), (2, 1, SINK_FIXED)])
def test_fixed_noise_cache_oracle_matches_scalar_brute_force(window, j, sink_mode):
    cfg = _clean_cfg(window_blocks=window, sink_mode=sink_mode, cache_mode=CACHE_FIXED_STEP, cache_step=j)
    wl = Workload("brute-fixed", cfg, 16, 5, 0.25)
    W = make_weights(wl)
    noises = [block_noise(wl, b) for b in range(wl.num_blocks)]
    from _brute import BruteStream
    bs = BruteStream(cfg, W)
    bs.set_sink(W.sink)
    want = bs.run_sequential_fixed(noises, j)
    s = OracleStream(cfg, W)
    s.set_sink(W.sink)
    for b in range(wl.num_blocks):
        out, fin = s.denoise_step(noises[b])
        assert fin == b
        np.testing.assert_allclose(out, np.array(want[b]), rtol=1e-11, atol=1e-11)


def test_fixed_noise_cache_is_timestep_forcing_without_a_window_and_differs_with_one():
    """Window 0: no step reads another block, so the fixed-noise cache computes the
    timestep-forced latents exactly; with a window the prior blocks come from another
    step's K/V and the latents differ."""
    for window, same in ((0, True), (1, False)):
        outs = {}
        for mode in (CACHE_TIMESTEP, CACHE_FIXED_STEP):
            cfg = _clean_cfg(window_blocks=window, cache_mode=mode, cache_step=2)
            wl = Workload("fx", cfg, 17, 4, 0.25)
            W = make_weights(wl)
            s = OracleStream(cfg, W)
            s.set_sink(W.sink)
            outs[mode] = [s.denoise_step(block_noise(wl, b))[0] for b in range(wl.num_blocks)]
        for b, (a, c) in enumerate(zip(outs[CACHE_TIMESTEP], outs[CACHE_FIXED_STEP])):
            if same or b == 0:
                # equal up to summation order (a masked key of weight 0 can join the product)
                np.testing.assert_allclose(a, c, rtol=1e-12, atol=1e-12)
            else:
                assert np.abs(a - c).max() > 1e-6


def test_fixed_noise_cache_window_reads_the_fixed_step_ring():
    cfg = _clean_cfg(window_blocks=2, cache_mode=CACHE_FIXED_STEP, cache_step=1)
    ts = TickScheduler(cfg)
    for b in range(5):
        run, fin = ts.begin_tick(True)
        for i, bb in run:
            assert ts.window_blocks(i, bb) == list(range(max(0, bb - 2), bb))
            assert ts.window_ring(i) == 1 and ts.ring_of(i) == i
            ts.append(i, bb)
        ts.end_tick(fin)
    with pytest.raises(ValueError):
        TickScheduler(_clean_cfg(cache_mode=CACHE_FIXED_STEP, cache_step=4))
    with pytest.raises(ValueError):
        TickScheduler(_clean_cfg(cache_mode=CACHE_FIXED_STEP, schedule=SCHED_PIPELINED))
