"""Host-side helpers for running the path on several GPUs (one process each).

The attention of every (batch, head, query block) is independent, so the path
shards with no exchange on the data path: each rank either processes its own
batch (weak scaling, what ``bench.py`` times) or a contiguous share of the
(batch, head) pairs of one job (``shard_pairs``).  The only collective is the
max over ranks of the measured device times.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_pairs(B: int, H: int, rank: int, world: int):
    """Contiguous share of the B*H (batch, head) pairs for ``rank``: (start, stop)."""
    total = B * H
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity on one rank)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device=None):
    """Element-wise sum of a list of floats over all ranks."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def job_throughput(flops_per_rank: float, ms_per_step_per_rank: float, device=None):
    """Whole-job TFLOP/s: flops summed over ranks / the slowest rank's time."""
    (total,) = sum_over_ranks([flops_per_rank], device)
    (t_max,) = max_over_ranks([ms_per_step_per_rank], device)
    return total / (t_max * 1e-3) / 1e12, t_max
