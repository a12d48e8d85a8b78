"""The benchmark's reference arm (the oracle on the host cores) and its JSON line,
run on CPU: the keys and values the line must carry, and the rank rule under a
multi-process launch (only rank 0 works and prints)."""
from __future__ import annotations

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, "bench.py", *args], capture_output=True, text=True,
                          cwd=ROOT, env=env, timeout=300)


def _check_line(d, unit):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["unit"] == unit and d["value"] > 0
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["data"] == "synthetic" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"] and cb["unit"] == unit
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == unit
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_linear_line():
    out = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
                  "--ref-budget-s", "1"])
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    _check_line(d, "TFLOP/s")
    assert d["config"]["workload"] == "tiny" and d["steps"] == 2 and d["warmup"] == 3


def test_reference_arm_kv_line():
    out = _bench(["--impl", "reference", "--path", "kv", "--kv-tokens", "64", "--steps", "1",
                  "--warmup", "3", "--ref-budget-s", "1"])
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), "GB/s")


def test_reference_arm_other_ranks_exit_quietly():
    out = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                 {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    out = _bench(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2"])
    assert out.returncode != 0 and "warmup" in out.stderr
