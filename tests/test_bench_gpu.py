"""The benchmark harness end to end on the GPU: one short run of the default
step with the extra report of every other workload, checked for the keys
the JSON line promises."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

import bench

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                         timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_default_step_line_with_extras():
    d = _line(["--steps", "2", "--warmup", "3", "--no-e2e", "--no-cpu-baseline"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "dtype", "data", "config", "roofline", "gpu_launches", "clocks", "kernels", "extras"):
        assert k in d, k
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["gpu_launches"] == 6 * 2
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and 0 < r["frac"] and r["achieved"] > 0
    assert set(d["extras"]) == set(bench.EXTRA_CONFIGS)
    for label, ex in d["extras"].items():
        assert ex["calls"], label
        for name, c in ex["calls"].items():
            assert c["us"] > 0 and c["gb_s"] > 0, (label, name)
