"""Host-side multi-process helpers (one process per GPU, torch.distributed).

The decode path partitions into independent (sequence, KV head, split) units,
so ranks shard sequences and need no collective on the data path; the only
collectives are the timing barrier and the max-over-ranks reduction of the
timed region.  Everything here also runs on the `gloo` backend on CPU.
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def rank_env() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 120) -> None:
    """Initialise the default process group with a short timeout, so ranks
    that wait for a missing peer fail instead of hanging."""
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def shard(n_items: int, rank: int, world: int) -> range:
    """Contiguous share of n_items for this rank (sizes differ by at most 1)."""
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return units_per_rank * world * steps / (max_ms / 1e3)
