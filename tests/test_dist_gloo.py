"""The multi-rank host logic on CPU: two gloo ranks on 127.0.0.1.

Covers what `bench.py --gpus N` relies on besides the GPU: the slowest
rank's time, the whole-job throughput, and the adapter-gradient all-reduce
(the data-parallel exchange step) over a flat buffer with per-layer views.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from host_streamed_nf4_b200 import dist as hdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank "took" a different time; the job time is the max
        ms = 10.0 + 5.0 * rank
        ms_max = hdist.max_over_ranks(ms)
        value = hdist.job_throughput(512, 20, ms_max, ws)
        # flat gradient buffer with views, as the stack lays out dA/dB
        flat = torch.zeros(3 * 4 + 5 * 4)
        dA, dB = flat[:12].view(3, 4), flat[12:].view(5, 4)
        dA.fill_(rank + 1.0)
        dB.copy_(torch.arange(20, dtype=torch.float32).view(5, 4) * (rank + 1))
        hdist.allreduce_grads(flat)
        q.put((rank, ms_max, value, dA.clone(), dB.clone()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_throughput_and_grad_allreduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value, dA, dB in results:
        assert ms_max == 15.0
        assert abs(value - 2 * 512 * 20 / 0.015) < 1e-6 * value
        assert torch.equal(dA, torch.full((3, 4), 3.0))  # 1 + 2
        assert torch.equal(dB, torch.arange(20, dtype=torch.float32).view(5, 4) * 3)


def test_single_rank_is_identity():
    assert hdist.world() == (1, 0)
    assert hdist.max_over_ranks(7.5) == 7.5
    flat = torch.ones(4)
    hdist.allreduce_grads(flat)
    assert torch.equal(flat, torch.ones(4))
    assert hdist.job_throughput(512, 10, 1000.0, 1) == 5120.0


# ---------------------------------------------------------------- sharded stream

def test_shard_ranges_tile_every_block():
    from host_streamed_nf4_b200 import hsnf4
    for B in (1, 500, 1024, 1025, 5000, 131088384, 3 * 1024 * 1024 + 7):
        for world in (1, 2, 3, 4, 8):
            spans = [hsnf4.shard_range(B, world, r) for r in range(world)]
            S = spans[0][0]
            assert S % 1024 == 0 and world * S >= B and (S - 1024) * world < B
            covered = 0
            for r, (s_, off, n) in enumerate(spans):
                assert s_ == S and off == r * S
                assert n == max(0, min(S, B - off))
                covered += n
            assert covered == B


def test_shard_slabs_hold_exactly_each_ranks_shards():
    """The shard slabs of a node's ranks, between them, hold every byte of the
    stack exactly once: each rank's slab is its shard of every block, packed
    block after block."""
    from host_streamed_nf4_b200 import hsnf4
    descs = [hsnf4.layer_desc([(896, 1024), (128, 1024), (1024, 1536), (1024, 512)])] * 7
    full = hsnf4.slab_bytes(descs)
    layer = hsnf4.layer_bytes(descs[0])
    for bs in (1, 2, 3, 4, 7):
        n_blocks = (7 + bs - 1) // bs
        for world in (1, 2, 3, 4, 8):
            totals = 0
            for rank in range(world):
                layout, total = hsnf4.shard_slab_layout(descs, bs, world, rank)
                assert len(layout) == n_blocks
                at = 0
                for b, (off, n) in enumerate(layout):
                    B = (min(7, (b + 1) * bs) - b * bs) * layer
                    assert (off, n) == (at, hsnf4.shard_range(B, world, rank)[2])
                    at += n
                assert at == total
                totals += total
            assert totals == full, (bs, world)


def _gather_worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from host_streamed_nf4_b200 import hsnf4
        g = torch.Generator().manual_seed(5)
        slab = torch.randint(0, 256, (20000,), dtype=torch.uint8, generator=g)  # same on all ranks
        results = []
        for B, slot_off in ((5000, 0), (500, 8192), (20000, 0)):
            S, off, n = hsnf4.shard_range(B, ws, rank)
            ring = torch.zeros(2 * ws * S + 8192, dtype=torch.uint8)
            # this rank's shard lands at its offset, as the streamer's copy puts it
            ring[slot_off + off: slot_off + off + n] = slab[off: off + n]
            hdist.ring_gather(ring)(slot_off, S, ws, 0)
            results.append(bool(torch.equal(ring[slot_off: slot_off + B], slab[:B])))
        # a stack whose ranks each hold only their shard slab: every block
        # rebuilt through the gather equals the block of the whole stack
        descs = [hsnf4.layer_desc([(384, 512), (128, 512)])] * 5
        full = torch.randint(0, 256, (hsnf4.slab_bytes(descs),), dtype=torch.uint8, generator=g)
        layer = hsnf4.layer_bytes(descs[0])
        bs = 2
        layout, total = hsnf4.shard_slab_layout(descs, bs, ws, rank)
        mine = torch.empty(total, dtype=torch.uint8)
        for b, (at, n) in enumerate(layout):
            B = (min(5, (b + 1) * bs) - b * bs) * layer
            _, off, n2 = hsnf4.shard_range(B, ws, rank)
            mine[at: at + n] = full[b * bs * layer + off: b * bs * layer + off + n2]
        for b, (at, n) in enumerate(layout):
            B = (min(5, (b + 1) * bs) - b * bs) * layer
            S, off, _ = hsnf4.shard_range(B, ws, rank)
            ring = torch.zeros(ws * S, dtype=torch.uint8)
            ring[off: off + n] = mine[at: at + n]
            hdist.ring_gather(ring)(0, S, ws, b)
            results.append(bool(torch.equal(ring[:B], full[b * bs * layer: b * bs * layer + B])))
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


def test_ring_gather_rebuilds_the_block_on_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok in results:
        assert all(ok), (rank, ok)
