"""bench.py's reference arm on the host cores: one JSON line on rank 0 with
the oracle's throughput and how it was sampled; nothing on other ranks."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(rank, world):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
               MASTER_ADDR="127.0.0.1", MASTER_PORT="29555")
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                           "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_line_on_rank0():
    r = _run(0, 1)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "warm-up" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("decode step T=8")
    # The reference arm describes the workload exactly as the GPU arm's line
    # does (both build it with bench.workload_config), so the two lines' configs
    # compare equal.
    sys.path.insert(0, ROOT)
    import bench
    assert d["config"] == bench.workload_config(bench.parse(["--steps", "1", "--warmup", "3"]), "decode", 1)
    assert set(d["config"]) == {"workload", "tokens_per_step_per_gpu", "layers_rotated", "l2", "parallelism"}


def test_reference_arm_other_ranks_print_nothing():
    r = _run(1, 2)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
