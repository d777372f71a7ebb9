"""Host-side multi-GPU plumbing for the benchmark: one process per GPU.

The decode path shards by (batch, kv-head) unit with no data exchange, so
ranks never communicate on the data path: each rank serves its own batch of
sequences (weak scaling).  The only collectives are the timing reductions
below, taken outside the timed region.
"""
from __future__ import annotations

import os


def rank_info():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def workload_seed(rank: int, base: int = 0) -> int:
    """Each rank's batch is an independent draw of the same workload."""
    return base + rank


def _reduce(x: float, op, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def reduce_max(x: float, device=None) -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.MAX, device)


def reduce_sum(x: float, device=None) -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.SUM, device)


def aggregate_throughput(units_per_rank: float, ms_per_step_per_rank: float, device=None):
    """Whole-job rate: all ranks' units divided by the slowest rank's time."""
    total = reduce_sum(units_per_rank, device)
    ms = reduce_max(ms_per_step_per_rank, device)
    return total / (ms / 1e3), ms, total
