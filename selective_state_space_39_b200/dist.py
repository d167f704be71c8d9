"""Multi-GPU plumbing for the scan: it shards with no data-path collective.

Every (batch, channel) row of the selective scan is independent (the §3.3
recurrence runs along the sequence only), so N GPUs each take their own
slice of the batch. The only collectives are the timing barrier and the
max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def batch_shard(global_batch: int, world_size: int, rank: int):
    """(start, count) of the batch rows rank `rank` owns: contiguous, sizes
    differing by at most one, covering 0..global_batch exactly once."""
    if world_size < 1 or not 0 <= rank < world_size or global_batch < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(global_batch, world_size)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def env_world():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0):
    """Initialise the default process group when WORLD_SIZE > 1."""
    rank, _, world = env_world()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier(device=None):
    if dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (the rank itself when alone)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def finish():
    if dist.is_initialized():
        dist.destroy_process_group()
