"""Data-parallel plumbing for the streamed LoRA stack (torch.distributed).

Each rank runs the same layers on its own micro-batch (its own tokens).  The
one exchange step of data-parallel LoRA training is the sum of the adapter
gradients over ranks, once per step; the stack keeps every dA/dB in one flat
fp32 buffer so that this is a single all-reduce.  Timing takes the slowest
rank.

Sharded streaming: the ranks of a node stream the same frozen base, so each
rank copies only 1/world of every block over its own PCIe link and an
in-place all-gather (NVLink through NCCL) rebuilds the block in every rank's
ring slot, cutting per-GPU PCIe bytes world-fold.  `ring_gather` is the
callback the streamer calls for it.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(), dist.get_rank()
    return 1, 0


def _reduce_device() -> torch.device:
    # NCCL reduces CUDA tensors; gloo reduces CPU tensors
    if dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def max_over_ranks(x: float) -> float:
    """The largest value of x over all ranks (x itself without a group)."""
    ws, _ = world()
    if ws == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, ms_max: float, ws: int) -> float:
    """Whole-job units per second: every rank processed units_per_rank_step
    per step, and the job took the slowest rank's time."""
    return ws * units_per_rank_step * steps / (ms_max / 1e3)


def allreduce_grads(flat: torch.Tensor) -> None:
    """Sum the flat adapter-gradient buffer over ranks in place (the data-
    parallel exchange step); a no-op on one rank."""
    ws, _ = world()
    if ws > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)


def ring_gather(ring: torch.Tensor, group=None):
    """The streamer's gather callback for a ring tensor: the in-place
    all-gather of ring[slot_off, slot_off + world * shard_bytes), where this
    rank's shard is already in place at rank * shard_bytes.  Runs on the
    current stream (the streamer enters its copy stream first).  NCCL uses
    the in-place all-gather; gloo (CPU) the list form into views."""
    rank = dist.get_rank(group)
    nccl = dist.get_backend(group) == "nccl"

    def gather(slot_off: int, shard_bytes: int, world: int, block: int) -> None:
        out = ring[slot_off: slot_off + world * shard_bytes]
        mine = out[rank * shard_bytes: (rank + 1) * shard_bytes]
        if nccl:
            dist.all_gather_into_tensor(out, mine, group=group)
        else:
            dist.all_gather(list(out.split(shard_bytes)), mine.clone(), group=group)

    return gather
