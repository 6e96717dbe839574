"""The library's tick scheduler on the host (la_sched_trace, no GPU) against the
oracle's TickScheduler (oracle/schedule.py), call by call.

Every integer of the index state must agree: the tick and block counters, the
sink generation, each slot's block, ring entry, evicted block, sink and frame
temporal positions, and every ring's resident blocks and (block, step) tags.
The GPU tests check the same state from real streams; here the scheduler runs
alone over long call sequences, pipeline bubbles and drains included, for each
schedule and cache mode.
"""
import numpy as np
import pytest

from oracle.schedule import TickScheduler
from workloads import (CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP, SCHED_PIPELINED, SCHED_SEQUENTIAL, SINK_AAS,
                       SINK_FIXED, TINY)


def _oracle_states(cfg, has_new):
    sc = TickScheduler(cfg)
    states = []
    for nw in has_new:
        run, finished = sc.begin_tick(bool(nw))
        for i, b in run:
            sc.append(i, b)
        if sc.clean and finished >= 0:
            sc.append_refresh(finished)
        sc.end_tick(finished)
        states.append(sc.index_state())
    return np.stack(states)


def _trace(cfg, has_new):
    from streaming_causal_video_timestep_b200 import sched_trace
    return sched_trace(cfg, has_new)


def _pattern(seed, n, p_new):
    rng = np.random.default_rng(seed)
    return [1] + [int(x) for x in (rng.random(n - 1) < p_new)]


PIPELINED = [
    dict(window_blocks=2, sink_mode=SINK_AAS),
    dict(window_blocks=0, sink_mode=SINK_AAS),
    dict(window_blocks=8, sink_mode=SINK_FIXED),
    dict(window_blocks=3, sink_mode=SINK_AAS, rolling_rope=0),
    dict(window_blocks=2, sink_mode=SINK_AAS, frames_per_block=5, sink_offset_frames=7),
    dict(window_blocks=1, sink_mode=SINK_AAS, timesteps=(1.0, 0.5, 0.0)),
    dict(window_blocks=2, sink_mode=SINK_FIXED, timesteps=(1.0, 0.8, 0.6, 0.4, 0.3, 0.2, 0.1, 0.0)),
]


@pytest.mark.parametrize("over", PIPELINED)
@pytest.mark.parametrize("p_new", [1.0, 0.7])
def test_pipelined_scheduler_matches_oracle(over, p_new):
    """Every call of a 200-call stream: steady blocks, or with bubbles (calls
    without a new block), ending with a drain of num_steps - 1 empty calls."""
    cfg = TINY.cfg.replace(schedule=SCHED_PIPELINED, **over)
    has_new = _pattern(7, 200, p_new) + [0] * (cfg.num_steps - 1)
    np.testing.assert_array_equal(_trace(cfg, has_new), _oracle_states(cfg, has_new))


@pytest.mark.parametrize("over", [
    dict(window_blocks=2, sink_mode=SINK_AAS),
    dict(window_blocks=0, sink_mode=SINK_FIXED),
    dict(window_blocks=2, sink_mode=SINK_AAS, cache_mode=CACHE_CLEAN_REFRESH),
    dict(window_blocks=1, sink_mode=SINK_FIXED, cache_mode=CACHE_CLEAN_REFRESH),
    dict(window_blocks=2, sink_mode=SINK_AAS, cache_mode=CACHE_FIXED_STEP, cache_step=3),
    dict(window_blocks=3, sink_mode=SINK_FIXED, cache_mode=CACHE_FIXED_STEP, cache_step=0),
])
def test_sequential_scheduler_matches_oracle(over):
    cfg = TINY.cfg.replace(schedule=SCHED_SEQUENTIAL, **over)
    has_new = [1] * 120
    np.testing.assert_array_equal(_trace(cfg, has_new), _oracle_states(cfg, has_new))


def test_long_stream_counters_and_rings():
    """10,000 calls: the counters and the ring contents stay exact (the GPU soak's
    index state, without the passes)."""
    cfg = TINY.cfg.replace(schedule=SCHED_PIPELINED, window_blocks=2, sink_mode=SINK_AAS)
    has_new = [1] * 10000 + [0] * (cfg.num_steps - 1)
    got = _trace(cfg, has_new)
    np.testing.assert_array_equal(got[::997], _oracle_states(cfg, has_new)[::997])
    np.testing.assert_array_equal(got[-1][:4], [len(has_new) - 1, 10000, 10000, 1])


def test_sequential_call_without_a_block_is_a_state_error():
    from streaming_causal_video_timestep_b200 import LaError
    cfg = TINY.cfg.replace(schedule=SCHED_SEQUENTIAL)
    with pytest.raises(LaError):
        _trace(cfg, [1, 1, 0, 1])


@pytest.mark.parametrize("over", [dict(window_blocks=-1), dict(num_steps=0), dict(cache_mode=9),
                                  dict(schedule=SCHED_PIPELINED, cache_mode=CACHE_CLEAN_REFRESH)])
def test_bad_scheduling_configuration_is_rejected(over):
    from streaming_causal_video_timestep_b200 import LaError
    if "num_steps" in over:
        cfg = TINY.cfg.replace(timesteps=(1.0,))
    else:
        cfg = TINY.cfg.replace(**over)
    with pytest.raises(LaError):
        _trace(cfg, [1, 1])


@pytest.mark.parametrize("window,r", [(2, 0), (2, 3), (0, 1), (5, 2)])
def test_slot_schedule_follows_the_pipelined_slot(window, r):
    """A slot stream (LA_SCHED_SLOT, one rank of the timestep pipeline) keeps step r's
    ring exactly as slot r of the grouped pipelined stream does: its call k runs block
    k, as the pipelined stream's slot r does at call k + r."""
    from workloads import SCHED_SLOT
    n = 40
    base = TINY.cfg.replace(window_blocks=window, sink_mode=SINK_FIXED)
    S = base.num_steps
    slot = _trace(base.replace(schedule=SCHED_SLOT, slot_index=r), [1] * n)
    pipe = _trace(base.replace(schedule=SCHED_PIPELINED), [1] * (n + S - 1))
    per = 8 + 3 * base.ring_entries
    for k in range(n):
        a = slot[k][4 + r * per: 4 + (r + 1) * per]
        b = pipe[k + r][4 + r * per: 4 + (r + 1) * per]
        np.testing.assert_array_equal(a, b)
        assert a[0] == k
