"""Data-parallel plumbing for one process per GPU.

The mixer's sequences are independent, so N GPUs run N replicas of the whole
path, each on its own slice of the batch; the data path has no collective.
Across ranks there are only barriers and the timing reduction: a run's time is
the maximum of the ranks' device times, and its throughput is every rank's
tokens divided by that time (weak scaling: the batch per rank stays fixed).
"""
from __future__ import annotations

import datetime
from typing import Optional, Tuple


def shard(batch_per_rank: int, rank: int) -> Tuple[int, int]:
    """Sequences [lo, hi) of the global batch that ``rank`` owns."""
    if batch_per_rank < 0 or rank < 0:
        raise ValueError("batch_per_rank and rank must be non-negative")
    return rank * batch_per_rank, (rank + 1) * batch_per_rank


def init(backend: str, timeout_s: float = 120.0, device=None) -> None:
    """Join the process group described by RANK / WORLD_SIZE / MASTER_* with a
    short timeout, so that ranks stuck waiting for one another end with an error."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device: Optional[object] = None) -> float:
    """The maximum of ``value`` over all ranks (the value itself without a group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput (units per second) from the max-over-ranks time in ms."""
    if ms <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / (ms / 1e3)
