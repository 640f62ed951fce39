"""The pinned-host -> VRAM ring on the GPU.

The pages' correctness bar for streaming is bitwise identity with a
resident run, at any block_size ("Poros on consumer GPUs": NF4 is the
precision with 0.00e+00 parity to a fully resident run; block_size never
affects parity.  Poros API reference: elementwise-exact resident parity,
torch.equal).  These tests hold the ring to exactly that, plus its byte
accounting, lifetime fences and protocol errors.
"""
import pytest
import torch

from host_streamed_nf4_b200 import hsnf4, synth
from host_streamed_nf4_b200.stack import LayerStack

pytestmark = pytest.mark.gpu

TINY = synth.Family("tiny", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=6)


def _run(stack, steps=2):
    rec = {}

    def record(l, p, name, t):
        rec[(l, p, name)] = t.clone()

    for _ in range(steps):
        rec.clear()
        stack.step(record)
    torch.cuda.synchronize()
    assert hsnf4.device_status() == 0
    for l in range(stack.L):
        for p in range(stack.P):
            rec[(l, p, "t")] = stack.t[l][p].clone()
            rec[(l, p, "dA")] = stack.dA[l][p].clone()
            rec[(l, p, "dB")] = stack.dB[l][p].clone()
    return rec


def _assert_bitwise(a, b):
    assert a.keys() == b.keys()
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.fixture(scope="module")
def resident6():
    s = LayerStack(TINY, 6, 96, streamed=False)
    rec = _run(s)
    s.close()
    return rec


@pytest.mark.parametrize("bs,slots", [(1, 2), (2, 2), (4, 2), (1, 3), (2, 4)])
def test_streamed_equals_resident_bitwise(resident6, bs, slots):
    s = LayerStack(TINY, 6, 96, block_size=bs, streamed=True, n_slots=slots)
    rec = _run(s)
    s.close()
    _assert_bitwise(rec, resident6)


def test_partial_last_block_bitwise():
    res = LayerStack(TINY, 5, 64, streamed=False)
    a = _run(res)
    res.close()
    for bs in (2, 4):
        s = LayerStack(TINY, 5, 64, block_size=bs, streamed=True)
        _assert_bitwise(_run(s), a)
        s.close()


@pytest.mark.parametrize("bs,reuse,slots", [(1, True, 2), (2, True, 2), (4, True, 2),
                                             (1, False, 2), (2, False, 2), (1, True, 3),
                                             (1, True, 4), (2, True, 3)])
def test_h2d_bytes_match_the_schedule(bs, reuse, slots):
    s = LayerStack(TINY, 6, 32, block_size=bs, streamed=True, reuse_resident=reuse, n_slots=slots)
    s.step()
    s.step()
    before = s.streamer.stats()
    s.step()
    torch.cuda.synchronize()
    after = s.streamer.stats()
    moved = after["h2d_bytes"] - before["h2d_bytes"]
    assert moved == s.steady_h2d_bytes_per_step(reuse_resident=reuse, n_slots=slots)
    assert after["acquires"] - before["acquires"] == 2 * s.n_blocks
    assert after["releases"] - before["releases"] == 2 * s.n_blocks
    s.close()


def test_poisoned_release_still_bitwise(resident6):
    """A released slot is overwritten with 0xFF: any read after release would
    break the bitwise comparison."""
    s = LayerStack(TINY, 6, 96, block_size=2, streamed=True, poison_on_release=True)
    _assert_bitwise(_run(s), resident6)
    s.close()


def test_no_prefetch_mode_bitwise(resident6):
    s = LayerStack(TINY, 6, 96, block_size=2, streamed=True, enable_prefetch=False)
    _assert_bitwise(_run(s), resident6)
    s.close()


# ---------------------------------------------------------------- protocol

def _small_streamer(reuse=True, n_layers=4, bs=1, slots=2):
    descs = [hsnf4.layer_desc([(128, 256), (64, 128)])] * n_layers
    slab = torch.zeros(hsnf4.slab_bytes(descs), dtype=torch.uint8, pin_memory=True)
    ring = torch.empty(hsnf4.ring_bytes(descs, bs, slots), dtype=torch.uint8, device="cuda")
    cs = torch.cuda.Stream()
    return hsnf4.Streamer(slab, descs, bs, ring, cs, reuse_resident=reuse, n_slots=slots), cs


def _status(fn):
    with pytest.raises(hsnf4.HsNf4Error) as e:
        fn()
    return e.value.status


def test_protocol_misuse_is_reported():
    st, _ = _small_streamer()
    assert _status(lambda: st.release(0)) == hsnf4.ERR_STATE          # never acquired
    assert _status(lambda: st.acquire(1)) == hsnf4.ERR_STATE          # never prefetched
    assert _status(lambda: st.prefetch(4)) == hsnf4.ERR_INVALID       # out of range
    st.prefetch(0)
    st.prefetch(1)
    assert _status(lambda: st.prefetch(2)) == hsnf4.ERR_STATE         # two ahead: no free slot
    st.acquire(0)
    assert _status(lambda: st.acquire(0)) == hsnf4.ERR_STATE          # double acquire
    st.release(0)
    st.prefetch(2)                                                   # slot of block 0 is free now
    torch.cuda.synchronize()
    st.close()


def test_ring_too_small_is_oom_with_sizes():
    descs = [hsnf4.layer_desc([(128, 256)])] * 4
    slab = torch.zeros(hsnf4.slab_bytes(descs), dtype=torch.uint8, pin_memory=True)
    need = hsnf4.ring_bytes(descs, 2)
    ring = torch.empty(need - 1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(hsnf4.HsNf4Error) as e:
        hsnf4.Streamer(slab, descs, 2, ring, torch.cuda.Stream())
    assert e.value.status == hsnf4.ERR_OOM
    assert str(need) in e.value.detail and "block_size" in e.value.detail


def test_host_wait_times_out_then_succeeds():
    st, cs = _small_streamer()
    with torch.cuda.stream(cs):
        torch.cuda._sleep(400_000_000)  # keep the copy stream busy (~0.2 s)
    st.prefetch(0)
    assert _status(lambda: st.acquire_host(0, 1)) == hsnf4.ERR_TIMEOUT
    st.acquire_host(0, 20_000)
    torch.cuda.synchronize()
    st.close()


@pytest.mark.parametrize("site", ["copy_enqueue", "event_record"])
def test_injected_host_fault_leaves_streamer_usable(site):
    st, _ = _small_streamer()
    hsnf4.inject_fault(site)
    assert _status(lambda: st.prefetch(0)) == hsnf4.ERR_CUDA
    hsnf4.inject_fault(None)
    st.prefetch(0)  # retry works
    st.acquire(0)
    st.release(0)
    torch.cuda.synchronize()
    st.close()


def test_device_bounded_wait_gives_up_and_context_survives():
    """A kernel waits on a barrier nothing arrives at: the bounded wait gives
    up, records its flag, the kernel returns and the context stays usable."""
    assert hsnf4.device_status() == 0
    hsnf4.selftest_stall()
    flags = hsnf4.device_status()
    assert flags & 0x40
    assert hsnf4.device_status() == 0  # reading clears
    x = torch.arange(10, device="cuda").sum().item()
    assert x == 45


def test_prefetch_ahead_fills_free_slots_in_visit_order():
    st, _ = _small_streamer(n_layers=6)  # 2 slots
    assert st.prefetch_ahead([0, 1, 2]) == 2   # two free slots: blocks 0 and 1
    st.acquire(0)
    assert st.prefetch_ahead([1, 2, 3]) == 0   # 1 is already there; no free slot for 2
    st.release(0)
    assert st.prefetch_ahead([1, 2, 3]) == 1   # block 0's slot takes block 2
    torch.cuda.synchronize()
    assert st.stats()["copies"] == 3
    st.close()


# ---------------------------------------------------------------- sharded stream, one GPU

def _emulated_peers(holder, full_slab):
    """Gather factory that stands in for the other ranks on one GPU: it fills
    their shards of the slot from the whole stack's pinned slab (what their
    own PCIe copies would have brought), enqueued on the copy stream like the
    all-gather."""
    def factory(ring):
        def gather(slot_off, S, world, block):
            st = holder[0]
            B = st.block_bytes(block)
            base = block * st.block_size * st.layer_bytes
            for j in range(world):
                off = j * S
                n = max(0, min(S, B - off))
                if j != st.shard[0] and n:
                    ring[slot_off + off: slot_off + off + n].copy_(
                        full_slab[base + off: base + off + n], non_blocking=True)
        return gather
    return factory


@pytest.fixture(scope="module")
def tiny6_slab():
    s = LayerStack(TINY, 6, 96, streamed=False)
    slab = s.slab
    s.close()
    return slab


@pytest.mark.parametrize("world,rank,bs,shard_slab", [(2, 0, 1, True), (2, 1, 2, True),
                                                      (4, 3, 1, True), (4, 2, 4, True),
                                                      (2, 1, 2, False), (4, 2, 4, False)])
def test_sharded_stream_equals_resident_bitwise(resident6, tiny6_slab, world, rank, bs,
                                                shard_slab):
    holder = []
    s = LayerStack(TINY, 6, 96, block_size=bs, streamed=True,
                   shard=(rank, world, _emulated_peers(holder, tiny6_slab)), shard_slab=shard_slab)
    holder.append(s)
    if shard_slab:  # this rank pins only its shards: about 1/world of the stack
        assert s.pinned_bytes() < tiny6_slab.numel() / world + s.n_blocks * 1024
    _assert_bitwise(_run(s), resident6)
    st = s.streamer.stats()
    assert st["gathers"] == st["copies"] > 0
    # this rank's link moved only its shards
    before = s.streamer.stats()["h2d_bytes"]
    s.step()
    torch.cuda.synchronize()
    assert s.streamer.stats()["h2d_bytes"] - before == s.steady_h2d_bytes_per_step()
    # about 1/world of the unsharded bytes (shards are 1 KiB-rounded)
    full = sum(2 * s.block_bytes(b) for b in range(s.n_blocks))
    assert s.steady_h2d_bytes_per_step() <= full / world + 2 * s.n_blocks * 1024
    s.close()


def test_gather_failure_is_reported():
    def factory(ring):
        def gather(slot_off, S, world, block):
            raise RuntimeError("peer went away")
        return gather
    s = LayerStack(TINY, 2, 32, block_size=1, streamed=True, shard=(0, 2, factory))
    with pytest.raises(hsnf4.HsNf4Error) as e:
        s.step()
    assert e.value.status == hsnf4.ERR_CUDA and "peer went away" in str(e.value)
    torch.cuda.synchronize()
    s.close()


_NCCL_CHILD = r"""
import os, sys, datetime, torch
import torch.distributed as dist
sys.path.insert(0, os.environ["REPO"])
from host_streamed_nf4_b200 import dist as hdist, synth
from host_streamed_nf4_b200.stack import LayerStack
dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                        init_method="tcp://127.0.0.1:%s" % os.environ["PORT"],
                        device_id=torch.device("cuda", 0))
fam = synth.Family("tiny", hidden=256, inter=640, heads=2, kv_heads=1, head_dim=128, layers=4)
def run(st):
    out = []
    for _ in range(2):
        st.step()
    torch.cuda.synchronize()
    return [t.clone() for t in [st.grad_flat] + st.Y + st.dX]
ref = LayerStack(fam, 4, 64, streamed=False)
a = run(ref)
ref.close()
sh = LayerStack(fam, 4, 64, block_size=2, streamed=True, shard=(0, 1, hdist.ring_gather))
b = run(sh)
gathers = sh.streamer.stats()["gathers"]
sh.close()
ok = all(torch.equal(x, y) for x, y in zip(a, b)) and gathers > 0
dist.destroy_process_group()
print("NCCL_GATHER_OK" if ok else "NCCL_GATHER_MISMATCH")
"""


def test_nccl_ring_gather_on_one_rank():
    """The real NCCL gather path (in-place all_gather_into_tensor on the copy
    stream, called back from the streamer) with a one-rank process group."""
    import os
    import socket
    import subprocess
    import sys
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    repo = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, REPO=repo, PORT=str(port), NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _NCCL_CHILD], env=env, capture_output=True,
                       text=True, timeout=300)
    assert "NCCL_GATHER_OK" in r.stdout, (r.stdout[-2000:], r.stderr[-2000:])


@pytest.mark.parametrize("bs,dropout", [(2, 0.0), (4, 0.1)])
def test_resident_check_of_a_streamed_step(bs, dropout):
    """The bench's result check: layers 0 and L-1 recomputed from freshly
    drawn weights in VRAM equal the streamed step bit for bit."""
    s = LayerStack(TINY, 6, 96, block_size=bs, streamed=True, dropout=dropout)
    s.step()
    s.step()
    res = s.resident_check()
    s.close()
    assert res == {0: True, 5: True}
