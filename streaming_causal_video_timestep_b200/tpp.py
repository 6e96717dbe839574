"""The timestep-pipelined stream across devices (TPP): rank r owns denoising step r.

The papernotes note (关键设计 4) and the gitcode blog (question 6) describe the
system: each of num_steps GPUs is pinned to one step t_r -> t_{r+1} and keeps
that step's own noisy KV cache (timestep forcing), and only the latent moves
from GPU to GPU.  Here each rank holds a stream in the LA_SCHED_SLOT schedule
(one step of each block, with its own ring) and a tick is:

  1. rank 0 takes the next block's noise (or nothing, when draining); rank r > 0
     takes what rank r - 1 produced in the previous tick;
  2. a rank holding a block runs its step;
  3. it hands the latent (and the block's audio, for the DiT block's
     cross-attention) to rank r + 1; the last rank returns the finished block.
  4. (collective) the last rank tells every rank whether block 0 has just
     finished; if so, and the sink mode is the Adaptive Attention Sink, frame 0
     of it is broadcast and every rank replaces its sink before the next tick,
     the timing of the single-device pipeline.

The hand-off is the only data exchange: T_b x C fp32 (1.2 MB at the 14B-like
shape) plus a block id per rank and tick, and the sink frame once per stream.
Steps 1-3 run in TppRank.step, step 4 in TppRank.sync_sink, so a single
process can emulate the ranks (LocalTransport) by running step 1-3 of every
rank before step 4 of every rank.
"""
from __future__ import annotations

import torch


class DistTransport:
    """Point-to-point hand-off and the sink broadcast over torch.distributed (NCCL
    over NVLink on GPUs, gloo on the host).

    rank / world: the rank's step and the pipeline's length; base: the global
    rank of the pipeline's step 0 (several pipelines in one job each take a run
    of num_steps consecutive global ranks and their own process group, since
    torch.distributed addresses peers by global rank)."""

    def __init__(self, rank: int, world: int, device, group=None, base: int = 0):
        import torch.distributed as dist
        self.dist, self.rank, self.world, self.device, self.group = dist, rank, world, device, group
        self.base = base
        self._pending = []

    def send_next(self, tensors):
        # The previous tick's sends complete first; each send takes a copy, kept until
        # it completes, because the rank reuses its output buffer in the next tick.
        for w in self._pending:
            w.wait()
        self._keep = [t.contiguous().clone() for t in tensors]
        self._pending = [self.dist.isend(t, self.base + self.rank + 1, group=self.group) for t in self._keep]

    def recv_prev(self, shapes_dtypes):
        out = [torch.empty(s, dtype=d, device=self.device) for s, d in shapes_dtypes]
        for w in [self.dist.irecv(t, self.base + self.rank - 1, group=self.group) for t in out]:
            w.wait()
        return out

    def bcast_from_last(self, t):
        self.dist.broadcast(t, self.base + self.world - 1, group=self.group)
        return t

    def finish(self):
        for w in self._pending:
            w.wait()
        self._pending = []


class LocalTransport:
    """The ranks of one process: messages keyed by (sender, tick), broadcasts by
    (tick, call).  Used to run the TPP decomposition on one device: every rank's
    step, then sync_sink of the last rank first and of the others after it,
    tick by tick (run_local)."""

    def __init__(self, world: int):
        self.world = world
        self.box = {}
        self.bc = {}

    def endpoint(self, rank):
        return _LocalEnd(self, rank)


class _LocalEnd:
    def __init__(self, hub, rank):
        self.hub, self.rank = hub, rank
        self.tick = 0
        self._calls = {}

    def send_next(self, tensors):
        self.hub.box[(self.rank, self.tick)] = [t.clone() for t in tensors]

    def recv_prev(self, shapes_dtypes):
        return self.hub.box.pop((self.rank - 1, self.tick - 1))

    def bcast_from_last(self, t):
        n = self._calls.get(self.tick, 0)
        self._calls[self.tick] = n + 1
        if self.rank == self.hub.world - 1:
            self.hub.bc[(self.tick, n)] = t.clone()
        else:
            t.copy_(self.hub.bc[(self.tick, n)])
        return t

    def finish(self):
        pass


class TppRank:
    """One rank of the timestep pipeline.

    backend: the rank's slot stream; it provides T, C, step(x_in, x_out, audio=None)
    -> block id, replace_sink(latent) and the sink settings (LaStream in the
    LA_SCHED_SLOT schedule on a GPU).  transport: DistTransport or a
    LocalTransport endpoint.  audio_shape: (audio_tokens, audio_dim) for the DiT
    block's cross-attention, else None."""

    def __init__(self, backend, rank: int, world: int, transport, device, num_steps: int, sink_tokens: int,
                 aas: bool, audio_shape=None):
        if world != num_steps:
            raise ValueError("the timestep pipeline has one rank per denoising step")
        self.b, self.rank, self.world, self.tr, self.device = backend, rank, world, transport, device
        self.sink_tokens, self.aas, self.audio_shape = sink_tokens, aas, audio_shape
        self.tick_no = 0
        self.aas_done = not aas
        self._fin = None             # (block id, latent) the last rank finished this tick
        T, C = backend.T, backend.C
        self.x_out = torch.empty((T, C), dtype=torch.float32, device=device)

    def _message_layout(self):
        T, C = self.b.T, self.b.C
        lay = [((1,), torch.int64), ((T, C), torch.float32)]
        if self.audio_shape is not None:
            lay.append((tuple(self.audio_shape), torch.float32))
        return lay

    def step(self, x_new=None, audio=None):
        """Steps 1-3 of a tick.  Returns (finished block id, its latent) on the last rank
        when a block leaves the pipeline, else (-1, None)."""
        if hasattr(self.tr, "tick"):
            self.tr.tick = self.tick_no
        blk, x_in, au = -1, None, None
        if self.rank == 0:
            if x_new is not None:
                blk, x_in, au = 0, x_new, audio          # id: the slot stream counts its own blocks
        elif self.tick_no > 0:
            msg = self.tr.recv_prev(self._message_layout())
            if int(msg[0][0]) >= 0:
                blk, x_in = int(msg[0][0]), msg[1]
                au = msg[2] if self.audio_shape is not None else None
        done = -1
        if x_in is not None:
            done = self.b.step(x_in, self.x_out, audio=au) if self.audio_shape is not None \
                else self.b.step(x_in, self.x_out)
        if self.rank < self.world - 1:
            T, C = self.b.T, self.b.C
            msg = [torch.tensor([done], dtype=torch.int64, device=self.device),
                   self.x_out if done >= 0 else torch.zeros((T, C), dtype=torch.float32, device=self.device)]
            if self.audio_shape is not None:
                msg.append(au if (done >= 0 and au is not None)
                           else torch.zeros(tuple(self.audio_shape), dtype=torch.float32, device=self.device))
            self.tr.send_next(msg)
            self._fin = None
            return -1, None
        self._fin = (done, self.x_out.clone()) if done >= 0 else None
        return (done, self._fin[1]) if self._fin else (-1, None)

    def sync_sink(self):
        """Step 4 of a tick (collective over all ranks until the sink has been replaced)."""
        if not self.aas_done:
            flag = torch.zeros(1, dtype=torch.int64, device=self.device)
            if self.rank == self.world - 1 and self._fin is not None and self._fin[0] == 0:
                flag[0] = 1
            self.tr.bcast_from_last(flag)
            if int(flag[0]):
                C = self.b.C
                frame = torch.empty((self.sink_tokens, C), dtype=torch.float32, device=self.device)
                if self.rank == self.world - 1:
                    frame.copy_(self._fin[1][: self.sink_tokens])
                self.tr.bcast_from_last(frame)
                self.b.replace_sink(frame)
                self.aas_done = True
        self.tick_no += 1

    def tick(self, x_new=None, audio=None):
        fin = self.step(x_new, audio)
        self.sync_sink()
        return fin

    def close(self):
        """End of the stream on every rank: each rank after the first takes the last
        hand-off of its predecessor (the send of the final tick, which no later tick
        receives), then the rank's own sends are completed."""
        if hasattr(self.tr, "tick"):
            self.tr.tick = self.tick_no
        if self.rank > 0 and self.tick_no > 0:
            self.tr.recv_prev(self._message_layout())
        self.tr.finish()


def run_local(ranks, inputs):
    """Emulate the timestep pipeline in one process: ranks (TppRank objects on one
    LocalTransport, rank order), inputs: per tick the new block's (noise, audio)
    or None.  Returns {block id: finished latent} from the last rank."""
    done = {}
    for item in inputs:
        x_new, audio = item if item is not None else (None, None)
        for r in ranks:
            blk, lat = r.step(x_new if r.rank == 0 else None, audio if r.rank == 0 else None)
            if blk >= 0:
                done[blk] = lat
        for r in [ranks[-1]] + ranks[:-1]:
            r.sync_sink()
    return done
