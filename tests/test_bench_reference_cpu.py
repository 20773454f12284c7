"""bench.py's reference arm on CPU: `--impl reference` times the oracle on the
host cores and prints one JSON line with the contract's keys (no GPU)."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_prints_the_contract_line():
    d = _run("--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3 and d["gpu_launches"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("tiny")


def test_warmup_below_three_is_refused():
    env = dict(os.environ)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_graph_chunk_times_exactly_k_steps():
    # the timed pass replays a graph of `chunk` steps K / chunk times: chunk divides K, at most 20
    sys.path.insert(0, ROOT)
    import bench

    for k in (1, 2, 3, 7, 20, 21, 40, 97, 200, 300, 2000, 2001):
        c = bench.graph_chunk(k)
        assert 1 <= c <= 20 and k % c == 0, (k, c)
        assert all(k % d for d in range(c + 1, min(k, 20) + 1)), (k, c)   # the largest such divisor
    assert bench.graph_chunk(2000) == 20 and bench.graph_chunk(97) == 1 and bench.graph_chunk(3) == 3
