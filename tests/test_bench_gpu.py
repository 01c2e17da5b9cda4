"""The benchmark's own code path on a GPU: a short run of `bench.py` (the prefill step of
the 5120 -> 8192 layer, few steps, no extra legs) must exit 0 and print one JSON line
with the keys its consumers read."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_short_run_prints_its_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5", "--warmup", "3", "--no-extras",
           "--no-decoder", "--cpu-seconds", "1"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout[-2000:]
    r = json.loads(lines[0])
    # (the oracle baseline and the end-to-end leg belong to the extra legs this run skips)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "dtype", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in r, key
    assert r["steps"] == 5 and r["warmup"] == 3 and r["value"] > 0
    assert r["roofline"]["achieved"] > 0 and 0 < r["roofline"]["frac"] < 1.5
    assert r["gpu_launches"] > 0
