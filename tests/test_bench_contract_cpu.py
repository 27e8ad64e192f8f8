"""bench.py's reference arm (the oracle) runs on the CPU and prints the one
JSON line the contract asks for, for the step metric and for the
calibration fit."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def check_reference_line(d, steps, warmup):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["steps"] == steps and d["warmup"] == warmup and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_reference_arm_step_metric():
    d = run_bench("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1")
    check_reference_line(d, 2, 1)
    assert d["unit"] == "tokens/s" and d["config"]["workload"] == "tiny"


def test_reference_arm_calibration_fit():
    d = run_bench("--impl", "reference", "--config", "calibration_small", "--steps", "1",
                  "--warmup", "0", env_extra={"DSPARK_REF_SEQUENCES": "5000"})
    check_reference_line(d, 1, 0)
    assert d["unit"] == "entries/s" and d["config"]["N"] == 50_003 and d["config"]["K"] == 16
    assert d["config"]["requests"] == 5000


def test_gpus_two_without_launcher_starts_two_ranks():
    """`bench.py --gpus 2` with no launcher starts two ranks itself; the
    reference arm prints its one line on rank 0 and reports both ranks."""
    d = run_bench("--impl", "reference", "--gpus", "2", "--config", "tiny", "--steps", "1",
                  "--warmup", "0")
    assert d["impl"] == "reference" and d["n_gpus"] == 2
