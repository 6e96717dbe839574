"""The timestep-pipelined stream across devices (TPP): rank r owns denoising step r.

The papernotes note (关键设计 4) and the gitcode blog (question 6) describe the
system: each of num_steps GPUs is pinned to one step t_r -> t_{r+1} and keeps
that step's own noisy KV cache (timestep forcing), and only the latent moves
from GPU to GPU.  Here each rank holds a stream in the LA_SCHED_SLOT schedule
(one step of each block, with its own ring) and a tick is:

  1. (exchange) every rank hands what it produced in the previous tick (the
     latent, and the block's audio for the DiT block's cross-attention) to rank
     r + 1 and takes rank r - 1's, in one batched send / receive;
  2. rank 0 takes the next block's noise (or nothing, when draining); a rank
     holding a block runs its step; the last rank returns the finished block;
  3. (collective) the last rank tells every rank whether block 0 has just
     finished; if so, and the sink mode is the Adaptive Attention Sink, frame 0
     of it is broadcast and every rank replaces its sink before the next tick,
     the timing of the single-device pipeline.

Every send is matched by a receive of the same tick, before the tick's
collective, so no rank's send can wait on a peer that is itself waiting in the
collective (with a send at the end of the tick, received only in the next one,
a send that waits for its receiver and the broadcast queued behind it on the
same communicator could wait on each other across neighbours).

The hand-off is the only data exchange: T_b x C fp32 (1.2 MB at the 14B-like
shape) plus a block id per rank and tick, and the sink frame once per stream.
Steps 1-2 run in TppRank.step, step 3 in TppRank.sync_sink, so a single
process can emulate the ranks (LocalTransport) by running steps 1-2 of every
rank, in rank order, before step 3 of every rank.
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

    def exchange(self, send, recv_layout):
        """Send the tensors `send` to rank + 1 (None: nothing to send) and receive
        tensors of recv_layout [(shape, dtype), ...] from rank - 1 (None: nothing),
        as one batch; returns the received tensors (or None) once both are done."""
        ops, out = [], None
        if send is not None:
            ops += [self.dist.P2POp(self.dist.isend, t.contiguous(), self.base + self.rank + 1, group=self.group)
                    for t in send]
        if recv_layout is not None:
            out = [torch.empty(s, dtype=d, device=self.device) for s, d in recv_layout]
            ops += [self.dist.P2POp(self.dist.irecv, t, self.base + self.rank - 1, group=self.group) for t in out]
        if ops:
            for w in self.dist.batch_isend_irecv(ops):
                w.wait()
        return out

    def bcast_from_last(self, t):
        self.dist.broadcast(t, self.base + self.world - 1, group=self.group)
        return t


class LocalTransport:
    """The ranks of one process: messages keyed by (sender, tick), broadcasts by
    (tick, call).  Used to run the TPP decomposition on one device: every rank's
    step in rank order (so a rank's exchange finds its predecessor's message of
    the same tick), then sync_sink of the last rank first and of the others
    after it, tick by tick (run_local); close() in rank order likewise."""

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

    def exchange(self, send, recv_layout):
        if send is not None:
            self.hub.box[(self.rank, self.tick)] = [t.clone() for t in send]
        return self.hub.box.pop((self.rank - 1, self.tick)) if recv_layout is not None else None

    def bcast_from_last(self, t):
        n = self._calls.get(self.tick, 0)
        self._calls[self.tick] = n + 1
        if self.rank == self.hub.world - 1:
            self.hub.bc[(self.tick, n)] = t.clone()
        else:
            t.copy_(self.hub.bc[(self.tick, n)])
        return t



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
        self._outbox = None          # this rank's message of the previous tick, handed on in the next
        T, C = backend.T, backend.C
        self.x_out = torch.empty((T, C), dtype=torch.float32, device=device)

    def _message_layout(self):
        T, C = self.b.T, self.b.C
        lay = [((1,), torch.int64), ((T, C), torch.float32)]
        if self.audio_shape is not None:
            lay.append((tuple(self.audio_shape), torch.float32))
        return lay

    def _exchange(self):
        """Step 1: hand the previous tick's message on and take the predecessor's."""
        send = self._outbox if self.rank < self.world - 1 else None
        recv = self._message_layout() if self.rank > 0 else None
        self._outbox = None
        return self.tr.exchange(send, recv)

    def step(self, x_new=None, audio=None):
        """Steps 1-2 of a tick.  Returns (finished block id, its latent) on the last rank
        when a block leaves the pipeline, else (-1, None)."""
        if hasattr(self.tr, "tick"):
            self.tr.tick = self.tick_no
        blk, x_in, au = -1, None, None
        msg = self._exchange() if self.tick_no > 0 else None
        if self.rank == 0:
            if x_new is not None:
                blk, x_in, au = 0, x_new, audio          # id: the slot stream counts its own blocks
        elif msg is not None and int(msg[0][0]) >= 0:
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
            # a copy: the next tick's step writes x_out again, after the exchange
            self._outbox = [t.clone() for t in msg]
            self._fin = None
            return -1, None
        self._fin = (done, self.x_out.clone()) if done >= 0 else None
        return (done, self._fin[1]) if self._fin else (-1, None)

    def sync_sink(self):
        """Step 3 of a tick (collective over all ranks until the sink has been replaced)."""
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
        """End of the stream on every rank: the final tick's messages, which no later
        tick takes, are exchanged once more (and dropped)."""
        if hasattr(self.tr, "tick"):
            self.tr.tick = self.tick_no
        if self.tick_no > 0:
            self._exchange()


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
