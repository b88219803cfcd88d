"""Multi-GPU plumbing of the decode step.

One process per GPU.  Sequences are independent, so the path shards by batch: every rank
decodes its own sequences and no collective touches the data path.  Collectives appear only
in the measurement (max over ranks of the device time)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_batch(global_batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous shard (first sequence, count) of ``global_batch`` sequences for ``rank``:
    the first ``global_batch % world`` ranks take one extra sequence."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Largest ``value`` over the ranks of the default process group (the value itself when
    no group is initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds
