"""Replica bookkeeping for several GPUs of one node (host side only).

The decode path does not shard: with N GPUs, N independent replicas decode
their own sequences and nothing is exchanged on the data path.  What crosses
ranks is timing: every rank's device-measured time is reduced to the maximum
(the job is as slow as its slowest replica), and the job's throughput counts
the tokens of all ranks over that time.
"""
from __future__ import annotations

import datetime
import os


def dist_env():
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 600):
    """Process group with a bounded timeout, so a rank that never joins ends the others with an error."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the value itself on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds_max
