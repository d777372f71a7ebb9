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


def _free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _spawned(rank: int, world: int, port: int, fn, args):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    rc = fn(*args)
    raise SystemExit(int(rc or 0))


def launch_local(world: int, fn, *args, timeout_s: float = 1800.0) -> int:
    """Run ``fn(*args)`` in ``world`` processes on this node, with the
    environment torchrun would set (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR
    127.0.0.1, MASTER_PORT); processes are spawned, not forked, so no CUDA
    state is inherited.  Returns 0 when every rank exits 0; otherwise the
    ranks still running are terminated and the first non-zero exit code is
    returned."""
    import time

    import torch.multiprocessing as mp
    if world < 1:
        raise ValueError("world must be >= 1")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_spawned, args=(r, world, port, fn, args)) for r in range(world)]
    for p in procs:
        p.start()
    deadline = time.monotonic() + timeout_s
    rc = 0
    for p in procs:
        p.join(max(0.0, deadline - time.monotonic()))
        if p.exitcode is None:
            rc = rc or 124  # timed out
        elif p.exitcode != 0:
            rc = rc or p.exitcode
        if rc:
            break
    for p in procs:
        if p.is_alive():
            p.terminate()
            p.join(10)
    return rc
