"""The timestep pipeline across ranks (streaming_causal_video_timestep_b200/tpp.py) on the host.

Every rank runs one denoising step of each block with its own cache; the latent
is handed from rank to rank, and the Adaptive Attention Sink is broadcast from
the last rank when block 0 finishes.  Here each rank's step is the oracle's slot
pass (a test double of the rank's LA_SCHED_SLOT stream), so the ranks'
composition can be checked against the oracle's single-process pipelined
stream: four gloo ranks over torch.distributed, and the same ranks emulated in
one process.  The hand-off carries fp32 latents, so the finished blocks agree
with the fp64 single-process stream to fp32 rounding.
"""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as tdist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(aas=True, audio=False, steps=4, seed=3):
    from workloads import BLOCK_DIT, SINK_AAS, SINK_FIXED, TINY, Workload
    cfg = TINY.cfg.replace(sink_mode=SINK_AAS if aas else SINK_FIXED)
    if steps == 2:
        cfg = cfg.replace(timesteps=(1.0, 0.5, 0.0))
    if audio:
        cfg = cfg.replace(block_kind=BLOCK_DIT, ffn_dim=96, audio_tokens=6, audio_dim=8)
    return Workload("tpp", cfg, seed, 6, TINY.w_std, TINY.head_std)


class OracleSlot:
    """A rank's step with the oracle: step slot_index of each block, its own cache."""

    def __init__(self, wl, W, rank):
        from oracle import OracleStream
        self.o = OracleStream(wl.cfg, W)
        self.o.set_sink(W.sink)
        self.rank, self.n = rank, 0
        self.T, self.C = wl.cfg.block_tokens, wl.cfg.latent_ch

    def step(self, x_in, x_out, audio=None):
        b, self.n = self.n, self.n + 1
        if audio is not None:
            self.o.audio[b] = audio.double().numpy()
        x = self.o.slot_pass(x_in.double().numpy(), b, self.rank)
        x_out.copy_(torch.from_numpy(x.astype(np.float32)))
        return b

    def replace_sink(self, latent):
        self.o.set_sink(latent.double().numpy())


def _single_process(wl, W):
    from oracle import OracleStream
    from workloads import block_audio, block_noise
    s = OracleStream(wl.cfg, W)
    s.set_sink(W.sink)
    au = getattr(wl.cfg, "audio_tokens", 0) > 0
    done = {}
    for k in range(wl.num_blocks + wl.cfg.num_steps - 1):
        nb = k < wl.num_blocks
        out, fin = s.denoise_step(block_noise(wl, k) if nb else None,
                                  audio=block_audio(wl, k) if (nb and au) else None)
        if fin >= 0:
            done[fin] = out
    return done


def _inputs(wl):
    from workloads import block_audio, block_noise
    au = getattr(wl.cfg, "audio_tokens", 0) > 0
    seq = []
    for k in range(wl.num_blocks + wl.cfg.num_steps - 1):
        if k < wl.num_blocks:
            seq.append((torch.from_numpy(block_noise(wl, k)),
                        torch.from_numpy(block_audio(wl, k)) if au else None))
        else:
            seq.append(None)
    return seq


@pytest.mark.parametrize("aas,audio", [(True, False), (False, False), (True, True)])
def test_tpp_emulated_in_one_process_matches_the_pipelined_stream(aas, audio):
    from streaming_causal_video_timestep_b200.tpp import LocalTransport, TppRank, run_local
    from workloads import make_weights
    wl = _workload(aas, audio)
    W = make_weights(wl)
    S = wl.cfg.num_steps
    hub = LocalTransport(S)
    ash = (wl.cfg.audio_tokens, wl.cfg.audio_dim) if audio else None
    ranks = [TppRank(OracleSlot(wl, W, r), r, S, hub.endpoint(r), "cpu", S, wl.cfg.sink_tokens, aas, ash)
             for r in range(S)]
    got = run_local(ranks, _inputs(wl))
    want = _single_process(wl, W)
    assert sorted(got) == list(range(wl.num_blocks))
    for b in range(wl.num_blocks):
        np.testing.assert_allclose(got[b].numpy(), want[b], rtol=2e-6, atol=2e-6)


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from streaming_causal_video_timestep_b200.tpp import DistTransport, TppRank
        from workloads import make_weights
        wl = _workload(True, False)
        W = make_weights(wl)
        S = wl.cfg.num_steps
        tr = DistTransport(rank, world, "cpu")
        me = TppRank(OracleSlot(wl, W, rank), rank, world, tr, "cpu", S, wl.cfg.sink_tokens, True)
        done = {}
        for item in _inputs(wl):
            x_new = item[0] if (item is not None and rank == 0) else None
            blk, lat = me.tick(x_new)
            if blk >= 0:
                done[blk] = lat.numpy().copy()
        me.close()
        tdist.barrier()
        if rank == world - 1:
            want = _single_process(wl, W)
            out["blocks"] = sorted(done)
            out["err"] = max(float(np.abs(done[b] - want[b]).max()) for b in want)
    finally:
        tdist.destroy_process_group()


def test_tpp_over_four_gloo_ranks_matches_the_pipelined_stream():
    world, port = 4, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out["blocks"] == list(range(6))
    assert out["err"] < 2e-6


def test_tpp_needs_one_rank_per_step():
    from streaming_causal_video_timestep_b200.tpp import LocalTransport, TppRank

    class _B:
        T, C = 4, 2
    with pytest.raises(ValueError):
        TppRank(_B(), 0, 3, LocalTransport(3).endpoint(0), "cpu", 4, 1, False)


def _pipelines_main(rank, world, steps, port, out):
    """world / steps pipelines of `steps` consecutive ranks in one job, each over its
    own process group (DistTransport's base rank), each with its own workload."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from streaming_causal_video_timestep_b200.tpp import DistTransport, TppRank
        from workloads import make_weights
        groups = [tdist.new_group(list(range(p * steps, (p + 1) * steps))) for p in range(world // steps)]
        pid, r = rank // steps, rank % steps
        wl = _workload(True, False, steps=steps, seed=3 + pid)
        W = make_weights(wl)
        tr = DistTransport(r, steps, "cpu", group=groups[pid], base=pid * steps)
        me = TppRank(OracleSlot(wl, W, r), r, steps, tr, "cpu", steps, wl.cfg.sink_tokens, True)
        done = {}
        for item in _inputs(wl):
            x_new = item[0] if (item is not None and r == 0) else None
            blk, lat = me.tick(x_new)
            if blk >= 0:
                done[blk] = lat.numpy().copy()
        me.close()
        tdist.barrier()
        if r == steps - 1:
            want = _single_process(wl, W)
            out[pid] = (sorted(done), max(float(np.abs(done[b] - want[b]).max()) for b in want))
    finally:
        tdist.destroy_process_group()


def test_tpp_two_gloo_ranks_aas_broadcast_matches_the_pipelined_stream():
    """Two ranks, two denoising steps: block 0 leaves the last rank at tick 1 and its
    frame 0 is broadcast before tick 2, the single-process pipeline's AAS timing."""
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_pipelines_main, args=(2, 2, port, out), nprocs=2, join=True)
    blocks, err = out[0]
    assert blocks == list(range(6))
    assert err < 2e-6


def test_tpp_two_pipelines_in_one_job_over_their_own_groups():
    """Four gloo ranks as two 2-step pipelines (global ranks 0-1 and 2-3), as bench.py
    runs 8 GPUs as two 4-step pipelines: each matches the oracle on its own workload."""
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_pipelines_main, args=(4, 2, port, out), nprocs=4, join=True)
    for pid in (0, 1):
        blocks, err = out[pid]
        assert blocks == list(range(6))
        assert err < 2e-6


class _RendezvousHub:
    """Ranks as threads, with the blocking semantics of a GPU communicator: a send
    completes only once its receiver has taken the message, and a broadcast only
    once every rank has reached it.  (gloo buffers its sends, so the gloo tests
    cannot show a send and a collective waiting on each other.)  Every wait is
    bounded: a protocol that deadlocks fails the test instead of hanging it."""

    def __init__(self, world, limit_s=20.0):
        import threading
        self.world, self.limit = world, limit_s
        self.cv = threading.Condition()
        self.links = {}                     # (sender, seq) -> message
        self.taken = set()
        self.bar = threading.Barrier(world, timeout=limit_s)
        self.slot = [None]

    def _wait(self, pred, what):
        if not self.cv.wait_for(pred, timeout=self.limit):
            raise TimeoutError(f"deadlock: {what}")

    def endpoint(self, rank):
        return _RendezvousEnd(self, rank)


class _RendezvousEnd:
    def __init__(self, hub, rank):
        self.hub, self.rank = hub, rank
        self.sent = self.recvd = 0

    def exchange(self, send, recv_layout):
        h, out = self.hub, None
        with h.cv:
            key = None
            if send is not None:                       # post the send (both halves of the batch are posted
                key = (self.rank, self.sent)           # before either is waited on)
                self.sent += 1
                h.links[key] = [t.clone() for t in send]
                h.cv.notify_all()
            if recv_layout is not None:
                want = (self.rank - 1, self.recvd)
                self.recvd += 1
                h._wait(lambda: want in h.links, f"rank {self.rank} receiving {want}")
                out = h.links.pop(want)
                h.taken.add(want)
                h.cv.notify_all()
            if key is not None:
                h._wait(lambda: key in h.taken, f"rank {self.rank} sending {key}")
        return out

    def bcast_from_last(self, t):
        h = self.hub
        if self.rank == h.world - 1:
            h.slot[0] = t.clone()
        h.bar.wait()
        if self.rank != h.world - 1:
            t.copy_(h.slot[0])
        h.bar.wait()
        return t


@pytest.mark.parametrize("aas", [True, False])
def test_tpp_completes_with_rendezvous_sends(aas):
    """The pipeline's protocol under unbuffered sends (rank threads, one batched
    exchange a tick before the sink broadcast) finishes every block and matches
    the single-process pipelined stream."""
    import threading

    from streaming_causal_video_timestep_b200.tpp import TppRank
    from workloads import make_weights
    wl = _workload(aas)
    W = make_weights(wl)
    S = wl.cfg.num_steps
    hub = _RendezvousHub(S)
    ranks = [TppRank(OracleSlot(wl, W, r), r, S, hub.endpoint(r), "cpu", S, wl.cfg.sink_tokens, aas)
             for r in range(S)]
    seq = _inputs(wl)
    done, errors = {}, []

    def run(r):
        try:
            for item in seq:
                x_new = item[0] if (item is not None and r.rank == 0) else None
                blk, lat = r.tick(x_new)
                if blk >= 0:
                    done[blk] = lat
            r.close()
        except Exception as e:      # noqa: BLE001 - reported below
            errors.append(f"rank {r.rank}: {type(e).__name__}: {e}")
            hub.bar.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in ranks]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    assert not any(t.is_alive() for t in threads)
    want = _single_process(wl, W)
    assert sorted(done) == list(range(wl.num_blocks))
    for b in range(wl.num_blocks):
        np.testing.assert_allclose(done[b].numpy(), want[b], rtol=2e-6, atol=2e-6)
