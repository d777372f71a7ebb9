"""The benchmark's reference arm (CPU only): it times the oracle on a bounded
sample of the GQA workload and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600,
                       env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]


def test_gpus_must_match_the_launched_world():
    """--gpus N under a launcher that started a different number of ranks is
    refused (the line would otherwise claim N GPUs for another count)."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode != 0
    assert "--gpus 2 but the launcher started 1 rank" in r.stderr


def test_step_graphs_run_exactly_the_requested_steps():
    """The timed region replays graphs of consecutive steps: whole chunks, then
    one graph of the rest, so exactly n steps run and every graph starts at
    cache copy 0 after a graph that ended at the last copy."""
    sys.path.insert(0, ROOT)
    import bench
    for copies in (2, 3, 5):
        chunk = copies * max(1, 64 // copies)
        assert chunk % copies == 0
        for n in (0, 1, 3, 20, chunk - 1, chunk, chunk + 1, 3 * chunk + 7, 11088):
            plan = bench.graph_plan(n, chunk)
            assert sum(plan) == n
            assert all(0 < m <= chunk for m in plan)
            assert all(m == chunk for m in plan[:-1])   # only the last graph is short
