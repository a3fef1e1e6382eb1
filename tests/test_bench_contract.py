"""The bench's JSON line, checked on the CPU through its reference arm (the
fp64 oracle timed on the host cores): one line, the keys and types the
benchmark contract names, and the multi-rank rule (ranks other than 0 exit 0
without printing)."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    r.wall_s = time.perf_counter() - t0
    return r


def test_reference_arm_line():
    r = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == "fkv_step chunk-steps/s per layer"
    assert d["unit"] == "chunk-steps/s per layer"
    assert isinstance(d["value"], (int, float)) and d["value"] > 0
    assert d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["ms_per_step"] > 0
    assert d["scaling"] in ("weak", "strong")
    assert d["vs_baseline"] is None
    assert d["dtype"] == "f64"
    assert d["config"]["workload"] == "tiny"
    # the same config object as the GPU arm prints for this workload
    sys.path.insert(0, ROOT)
    import bench
    import fkv_workloads as wl
    w = wl.get("tiny")
    assert d["config"] == bench.bench_config(w, w)
    # the timed steps fit inside the process's own wall time
    assert d["steps"] * d["ms_per_step"] / 1e3 <= r.wall_s
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "cpu_model" in cb
    assert cb["unit"] == d["unit"] and isinstance(cb["sample"], str) and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
