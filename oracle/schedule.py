"""Integer state of the stream: tick schedule, ring entries, positions, sink generation.

Timestep-forcing pipeline (10100.com article, TPP figure caption; papernotes
note, 关键设计 4; gitcode blog, question 6): worker i is pinned to the step
t_i -> t_{i+1} and keeps its own cache.  On one device the 4 workers become 4
slots of one tick: at tick k slot i holds the block that slot i-1 held at tick
k-1 and slot 0 takes the new block, so in an uninterrupted stream slot i runs
block k - i.  The block in the last slot is finished at the end of its tick.

Ring (readings of the rolling cache, gitcode blog question 1 table: only the
most recent N blocks are kept): each (layer, slot) ring has window+1 entries;
block b writes entry b mod (window+1), which evicts block b - window - 1.  The
block reads the resident blocks b-window .. b-1 oldest first, then itself.

Index-state record (int32), identical to the C-ABI's debug export:
  header  [tick, blocks_in, blocks_out, sink_generation]
  per slot i (num_steps records):
    [active_block, write_entry, evicted_block, sink_tpos, frame_tpos,
     sink_generation_used, step_index, n_resident,
     resident[E] (oldest -> newest, -1 padded), tags[E] x (block, step)]
active_block, write_entry and evicted_block are -1 and sink_tpos, frame_tpos,
sink_generation_used are 0 for a slot idle this tick; step_index is the slot
index; n_resident, resident and tags always describe the ring contents.

Clean-cache refresh (the ablation the method removes; papernotes note, 关键设计 2
and the NFE column of its inference-efficiency ablation, the paper's Table 3; gitcode blog, question 4 table): one cache of
clean K/V serves every step, so all slots share ring 0 (their records describe
it); after the last step of block b one more pass runs the stack on the
finished latent and overwrites block b's entry, tagged (b, num_steps).  Only
in the sequential schedule.

Fixed-noise cache (the other alternative to timestep forcing that the
papernotes note's key findings compare, the paper's Table 6: "fixed noise or
clean cache"; admirer.cn article: same-step memory against clean memory):
reading: the prior blocks a step reads come from the cache of one fixed step
j = cache_step, whatever the current step; every step still writes its own
cache and attends to its own block's current K/V.  Only in the sequential
schedule (in the grouped pipeline step j's pass of a later block would evict
an entry that another slot of the same launch reads).
"""
from __future__ import annotations

import numpy as np

from workloads import CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP, SCHED_PIPELINED, SINK_AAS


def index_state_layout(cfg):
    E = cfg.ring_entries
    per_slot = 8 + 3 * E
    return 4, per_slot, 4 + cfg.num_steps * per_slot


class TickScheduler:
    def __init__(self, cfg):
        if cfg.cache_mode in (CACHE_CLEAN_REFRESH, CACHE_FIXED_STEP) and cfg.schedule == SCHED_PIPELINED:
            raise ValueError("the clean-cache refresh and the fixed-noise cache run in the sequential schedule")
        if cfg.cache_mode == CACHE_FIXED_STEP and not 0 <= cfg.cache_step < cfg.num_steps:
            raise ValueError("cache_step must name one of the steps")
        self.cfg = cfg
        self.clean = cfg.cache_mode == CACHE_CLEAN_REFRESH
        self.fixed = cfg.cache_step if cfg.cache_mode == CACHE_FIXED_STEP else None
        S, E = cfg.num_steps, cfg.ring_entries
        self.S, self.E = S, E
        self.slots = [-1] * S          # block held by each slot after the last tick
        self.tick = -1
        self.blocks_in = 0
        self.blocks_out = 0
        self.sink_generation = 0
        self.tags = [[(-1, -1)] * E for _ in range(S)]
        self._records = [self._idle_record(i) for i in range(S)]

    # -- one tick ---------------------------------------------------------
    def begin_tick(self, has_new: bool):
        """Start a call.  Returns (run, finished): run = [(slot, block)] in
        execution order, finished = the block completed by this call or -1.
        The caller appends each (slot, block) with append() right before it
        computes that step."""
        S = self.S
        if self.cfg.schedule == SCHED_PIPELINED:
            new_block = self.blocks_in if has_new else -1
            slots = [new_block] + self.slots[:-1]
            run = [(i, b) for i, b in enumerate(slots) if b >= 0]
            finished = slots[S - 1]
            self.slots = slots
        else:
            if not has_new:
                raise ValueError("the sequential schedule needs a new block on every call")
            b = self.blocks_in
            run = [(i, b) for i in range(S)]
            finished = b
        self.tick += 1
        if has_new:
            self.blocks_in += 1
        self._records = [self._idle_record(i) for i in range(S)]
        return run, finished

    def end_tick(self, finished: int):
        """Close a call; returns True when the sink must be replaced now (AAS)."""
        if finished >= 0:
            self.blocks_out += 1
        if finished == 0 and self.cfg.sink_mode == SINK_AAS and self.sink_generation == 0:
            self.sink_generation = 1
            return True
        return False

    def ring_of(self, i: int) -> int:
        """The cache slot i writes (and reads its own block from): its own, or the one clean cache."""
        return 0 if self.clean else i

    def window_ring(self, i: int) -> int:
        """The cache slot i reads the prior blocks from: its own, the clean one, or step cache_step's."""
        return self.fixed if self.fixed is not None else self.ring_of(i)

    def append(self, i: int, b: int):
        """Ring append of block b at step i; returns the slot's record."""
        cfg, E = self.cfg, self.E
        ring = self.ring_of(i)
        e = b % E
        evicted = self.tags[ring][e][0]
        self.tags[ring][e] = (b, i)
        resident = self.resident(ring)
        rec = [b, e, evicted, self.sink_tpos(b), cfg.frames_per_block * b,
               self.sink_generation, i, len(resident)]
        rec = rec + self._pad(resident) + [v for tag in self.tags[ring] for v in tag]
        self._records[i] = rec
        return rec

    def append_refresh(self, b: int) -> int:
        """The refresh pass of block b rewrites its entry of the clean cache; returns the entry."""
        e = b % self.E
        self.tags[0][e] = (b, self.S)
        return e

    # -- queries ------------------------------------------------------------
    def resident(self, ring):
        return sorted(t[0] for t in self.tags[ring] if t[0] >= 0)

    def window_blocks(self, i, b):
        """Prior blocks block b reads at step i, oldest first."""
        return [x for x in self.resident(self.window_ring(i)) if b - self.cfg.window_blocks <= x < b]

    def sink_tpos(self, b: int) -> int:
        cfg = self.cfg
        if cfg.rolling_rope:
            return cfg.frames_per_block * b - cfg.sink_offset_frames
        return -cfg.sink_offset_frames

    def index_state(self) -> np.ndarray:
        head = [self.tick, self.blocks_in, self.blocks_out, self.sink_generation]
        body = []
        for i in range(self.S):
            rec = list(self._records[i])
            # ring-content fields always reflect the current ring
            ring = self.ring_of(i)
            rec[7] = len(self.resident(ring))
            rec[8:8 + self.E] = self._pad(self.resident(ring))
            rec[8 + self.E:] = [v for tag in self.tags[ring] for v in tag]
            body += rec
        return np.asarray(head + body, dtype=np.int32)

    def _pad(self, xs):
        return list(xs) + [-1] * (self.E - len(xs))

    def _idle_record(self, i):
        return [-1, -1, -1, 0, 0, 0, i, 0] + [-1] * self.E + [-1] * (2 * self.E)
