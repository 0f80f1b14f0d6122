"""Host-side checks of the benchmark's workload plans (no GPU): every
configuration names known call kinds, its algorithmic bytes follow the
per-element figures of the design table, and the step's bytes are the
documented 3,476,900,864."""
from __future__ import annotations

import pytest

import bench

KINDS = {"fwd", "bwd", "renorm", "project", "momentum", "norms", "bwd_scalar", "l2", "l2res", "slerp", "l2bwd",
         "l2resbwd", "slerpbwd", "gate", "swiglu", "qk"}


@pytest.mark.parametrize("config", sorted(set(bench.WORKLOADS) - {"long_rows"}))
def test_plans_are_well_formed(config):
    wg, ag, calls, copies = bench.plan(config, 0)
    assert copies >= 1 and calls
    names = [c[0] for c in calls]
    assert len(set(names)) == len(names)
    for name, kind, group in calls:
        assert kind in KINDS, kind
        assert (group in wg) != (group in ag), group
        segs, act = (wg[group], None) if group in wg else (None, ag[group])
        b = bench.call_bytes(kind, segs, act)
        r = bench.call_rows(kind, segs, act)
        assert b > 0 and r > 0


def test_step_bytes_and_per_element_figures():
    wg, ag, calls, _ = bench.plan("step", 0)
    segs, act = wg["model"], ag["x"]
    E = sum(s.w.size for s in segs)
    R = sum(s.rows for s in segs)
    assert (E, R) == (100_073_472, 114_944)
    got = {name: bench.call_bytes(kind, segs if group in wg else None, None if group in wg else act)
           for name, kind, group in calls}
    A = 16384 * 4096
    assert got == {"wn_forward": E * 6 + R * 4, "l2_rows": A * 4, "wn_backward": E * 10 + R * 8,
                   "l2_rows_residual": A * 6, "row_renorm": E * 8, "slerp_rows": A * 6 + 4096 * 4}
    assert sum(got.values()) == 3_476_900_864


def test_transposed_rows_count_output_channels():
    wg, _, calls, _ = bench.plan("gain", 0)
    conv = wg["conv1d"]
    assert all(s.w.shape == (1600, 6400) and s.transposed for s in conv)
    assert bench.call_rows("fwd", conv) == 12 * 6400          # unit rows = the stored columns
    assert bench.call_bytes("fwd", conv) == 12 * 1600 * 6400 * 6 + 12 * 6400 * 4


def test_long_rows_cover_both_long_classes():
    """The long-row report (drawn on the device) times two cluster-class
    calls and two two-pass calls, each larger than L2."""
    from l2_row_b200 import ds

    op = {"fwd": ds.DS_OP_WN_FORWARD, "slerp": ds.DS_OP_SLERP_ROWS}
    paths = [ds.ds_row_class(op[kind], cols)[0] for _, kind, _, cols in bench.LONG_CALLS]
    assert paths.count(ds.DS_PATH_CLUSTER) == 2 and paths.count(ds.DS_PATH_TWO_PASS) == 2
    for _, kind, rows, cols in bench.LONG_CALLS:
        import types

        act = types.SimpleNamespace(rows=rows, cols=cols)
        b = rows * cols * 6 + rows * 4 if kind == "fwd" else bench.call_bytes("slerp", act=act)
        assert b > 126 * 2 ** 20


def test_extras_cover_every_other_workload():
    """After the default step the bench reports every other workload."""
    assert set(bench.EXTRA_CONFIGS) == set(bench.WORKLOADS) - {"step"}
    assert len(bench.EXTRA_CONFIGS) == len(set(bench.EXTRA_CONFIGS))


def test_reference_arm_line():
    """bench.py --impl reference (the float64 oracle on the host cores) prints
    one JSON line with the reference arm's keys; no GPU is touched."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s" and d["value"] > 0
    assert d["dtype"] == "f64" and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
