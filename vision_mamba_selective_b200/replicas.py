"""Multi-GPU plumbing for the scan: replicas over independent batch items.

Every (batch item, channel) sequence of the scan is independent and B/C are per
(batch item, token), so splitting the batch across GPUs needs no exchange at all:
each rank runs the same kernels on its own items and no collective touches the data
path.  The only cross-rank traffic is host-side bookkeeping: a barrier around the
timed region and the maximum of the per-rank device times.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank_world():
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Create the default process group with a short timeout, so that ranks waiting on
    a rank that has gone away end with an error instead of hanging."""
    if dist.is_initialized():
        return
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def batch_slice(global_batch: int, rank: int, world: int) -> slice:
    """Contiguous share of ``global_batch`` items for ``rank`` (sizes differ by at most 1)."""
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of the inputs a rank draws in a weak-scaling run (every rank a full batch)."""
    return seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Largest ``value`` over all ranks (identity without a process group)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
