"""bench.py on the host: the reference arm (the oracle on the host cores) runs
without a GPU and prints one JSON line with the keys its consumers read."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line(oracle_lib):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["unit"] == "jets/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == "n128_p128"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_under_two_ranks(oracle_lib):
    """Launched as two ranks, only rank 0 runs the oracle and prints its line
    (n_gpus = 2); rank 1 exits 0 without output."""
    base = dict(os.environ, WORLD_SIZE="2", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1", MASTER_PORT="29531")
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"]
    r1 = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=dict(base, RANK="1"))
    assert r1.returncode == 0, r1.stderr[-2000:]
    assert not [ln for ln in r1.stdout.splitlines() if ln.startswith("{")]
    r0 = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=dict(base, RANK="0"))
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [json.loads(ln) for ln in r0.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
