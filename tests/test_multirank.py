"""World-size-2 gloo test (CPU) of the benchmark's multi-rank host logic:
per-rank workloads are independent draws, and the job rate is all ranks'
tokens over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    from datetime import timedelta
    from quantized_decode_attention_tq_b200 import dist as tqd
    from quantized_decode_attention_tq_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, lr, ws = tqd.rank_info()
        w = inputs.make("ragged", seed=tqd.workload_seed(r), seq=64, with_q=False)
        tokens = float(w.seq_lens.sum())
        ms = 2.0 + rank  # rank 1 is the slow one
        rate, ms_max, total = tqd.aggregate_throughput(tokens, ms)
        q.put((rank, (r, lr, ws), tokens, rate, ms_max, total, w.seq_lens.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, i0, t0, rate0, ms0, tot0, l0), (r1, i1, t1, rate1, ms1, tot1, l1) = res
    assert i0 == (0, 0, 2) and i1 == (1, 1, 2)
    assert l0 != l1                       # independent per-rank batches
    assert ms0 == ms1 == 3.0              # the slowest rank sets the time
    assert tot0 == tot1 == t0 + t1
    assert rate0 == rate1 == pytest.approx((t0 + t1) / 3e-3)


def _launched_worker(path, value):
    """A rank started by dist.launch_local: joins a gloo group from the
    environment the launcher set and reduces through the benchmark helpers."""
    import torch.distributed as dist
    from datetime import timedelta
    from quantized_decode_attention_tq_b200 import dist as tqd
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        r, lr, ws = tqd.rank_info()
        total = tqd.reduce_sum(value + r)
        mx = tqd.reduce_max(float(r))
        with open(f"{path}.{r}", "w") as f:
            f.write(f"{r} {lr} {ws} {total} {mx}")
    finally:
        dist.destroy_process_group()
    return 0


def _failing_worker(rank_to_fail):
    import os
    return 3 if int(os.environ["RANK"]) == rank_to_fail else 0


def test_launch_local_runs_every_rank_with_the_torchrun_environment(tmp_path):
    from quantized_decode_attention_tq_b200 import dist as tqd
    path = str(tmp_path / "out")
    assert tqd.launch_local(2, _launched_worker, path, 10.0, timeout_s=300) == 0
    got = sorted(open(f"{path}.{r}").read().split() for r in range(2))
    assert got == [["0", "0", "2", "21.0", "1.0"], ["1", "1", "2", "21.0", "1.0"]]


def test_launch_local_reports_a_failing_rank():
    from quantized_decode_attention_tq_b200 import dist as tqd
    assert tqd.launch_local(2, _failing_worker, 1, timeout_s=300) == 3
