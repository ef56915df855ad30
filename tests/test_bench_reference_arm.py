"""bench.py --impl reference on the CPU: the oracle arm prints one JSON line
with the contract's keys on rank 0, matching the GPU arm's metric and config,
and ranks other than 0 exit without work."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_line():
    lines = run(["--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "0"])
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert "sample" in cb and cb["unit"] == line["unit"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    cfg = line["config"]
    assert cfg["workload"].startswith("ttt_linear_mse_f32") and cfg["chunk"] == 16
    assert cfg["batch"] == 1 and cfg["heads"] == 2 and cfg["seq_len"] == 256


def test_other_ranks_print_nothing():
    lines = run(["--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "0"],
                {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert lines == []
