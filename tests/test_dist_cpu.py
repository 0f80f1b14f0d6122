"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Rows are independent, so N GPUs run N replicas of the step (weak scaling)
with no collective on the data path; the only exchange is the max of the
ranks' device timings.  These tests cover that exchange, the whole-job
aggregate, the per-rank seeding and the reference arm's rank-0-only rule.
"""
from __future__ import annotations

import contextlib
import io
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, out_dir: str) -> None:
    import datetime

    from l2_row_b200 import workloads as wl

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        # per-rank timings: the slowest rank decides every entry
        mx = bench.max_over_ranks(dist, [1.0 + rank, 5.0 - rank, 3.0], "cpu")
        # the step's inputs are seeded by rank: replicas work on different data
        x = wl.activations(rank, rows=8, cols=16).acts[0].x
        digests = [None] * WORLD
        dist.all_gather_object(digests, x.tobytes().hex())
        # the reference arm runs on rank 0 only: other ranks return silently
        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(type("A", (), {"warmup": 1, "steps": 1})(), rank, WORLD)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "distinct": len(set(digests)), "ref_out": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("dist")
    mp.start_processes(_rank_main, args=(_free_port(), str(out)), nprocs=WORLD, join=True, start_method="spawn")
    res = []
    for r in range(WORLD):
        with open(out / f"rank{r}.json") as f:
            res.append(json.load(f))
    return res


def test_max_over_ranks_is_elementwise_max(results):
    for r in results:
        assert r["max"] == [2.0, 5.0, 3.0]


def test_ranks_draw_different_inputs(results):
    assert all(r["distinct"] == WORLD for r in results)


def test_reference_arm_only_on_rank0(results):
    assert results[1]["ref_out"] == ""


def test_max_over_ranks_without_group():
    assert bench.max_over_ranks(None, [1, 2.5], "cpu") == [1.0, 2.5]


def test_whole_job_aggregate():
    # N replicas of B bytes in the slowest rank's time
    assert bench.whole_job_gbs(1, 10**9, 1.0) == pytest.approx(1000.0)
    assert bench.whole_job_gbs(8, 10**9, 2.0) == pytest.approx(4000.0)
