"""GPU parity, small cases: the tiny workload (W [64,128], X/R [32,128]) on
every row class, ragged and padded shapes with guard canaries, empty
segments, and exact aliasing.  Every comparison is against the float64
oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

PATHS = [ds.DS_PATH_AUTO, ds.DS_PATH_WARP, ds.DS_PATH_CTA, ds.DS_PATH_CLUSTER, ds.DS_PATH_TWO_PASS]
PATH_IDS = ["auto", "warp", "cta", "cluster", "two_pass"]


@pytest.fixture(scope="module")
def tiny():
    return wl.tiny(0)


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_tiny_all_ops(tiny, path):
    seg = tiny.weights[0]
    act = tiny.acts[0]
    eps = tiny.eps
    with ds.force_path(path):
        for out in ("f32", "bf16"):
            (o,) = gu.run_forward([seg], out, eps)
            gu.check_forward(seg, o, eps, out, what=f"forward {out}")
        (gw, gg), = gu.run_backward([seg], "f32", eps)
        gu.check_backward(seg, gw, gg, eps)
        segb = wl.WeightSeg("wb", seg.w, seg.g, wl.to_bf16_bits(seg.gy))
        (gw, gg), = gu.run_backward([segb], "bf16", eps)
        gu.check_backward(segb, gw, gg, eps, what="backward bf16 gy")
        (w,) = gu.run_renorm([seg], eps)
        gu.check_renorm(seg, w, eps)
        (y,) = gu.run_l2([act], eps, residual=False)
        gu.check_l2(act, y, eps, residual=False)
        (y,) = gu.run_l2([act], eps, residual=True)
        gu.check_l2(act, y, eps, residual=True)
        (h,) = gu.run_slerp([act], eps)
        gu.check_slerp(act, h, eps)


def test_tiny_radius_and_unit_mode(tiny):
    seg = tiny.weights[0]
    emb = wl.WeightSeg("emb", seg.w, seg.g, seg.gy, radius=float(np.sqrt(128.0)))
    unit = wl.WeightSeg("unit", seg.w, None, seg.gy)
    for s in (emb, unit):
        (o,) = gu.run_forward([s], "f32", 1e-6)
        gu.check_forward(s, o, 1e-6, "f32")
        (gw, gg), = gu.run_backward([s], "f32", 1e-6)
        gu.check_backward(s, gw, gg, 1e-6)
        (w,) = gu.run_renorm([s], 1e-6)
        gu.check_renorm(s, w, 1e-6)


RAGGED_COLS = [1, 3, 5, 7, 8, 13, 127, 129, 255, 257, 1000, 1023, 2049, 4097]


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_ragged_weight_rows_with_guards(path):
    rng = np.random.default_rng(21)
    eps = 1e-6
    with ds.force_path(path):
        for cols in RAGGED_COLS:
            rows = 37
            ld = ((cols + 7) // 8) * 8 + 8            # padded rows, 16-byte aligned for fp32 and bf16
            seg = wl.WeightSeg("r", wl.drifted_rows(rng, rows, cols, 0.5), wl.gains(rng, rows),
                               wl.normal_bf16(rng, (rows, cols)))
            w, _ = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            w.copy_(gu.dev_f32(seg.w))
            g = gu.dev_f32(seg.g)
            out, buf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
            ds.ds_wn_forward([ds.WSeg(w=w, gain=g, w_eff=out)], "bf16", eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(buf, rows, cols, ld, gu.CANARY_BF16), cols
            gu.check_forward(seg, out, eps, "bf16", what=f"forward cols={cols}")
            gw, gbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            gg = torch.empty(rows, device="cuda")
            gy, _ = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
            gy.copy_(gu.dev_bf16(seg.gy))
            ds.ds_wn_backward([ds.WSeg(w=w, gain=g, gy=gy, grad_w=gw, grad_g=gg)], "bf16", eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(gbuf, rows, cols, ld, gu.CANARY_F32), cols
            gu.check_backward(seg, gw, gg, eps, what=f"backward cols={cols}")
            wpad, wbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            wpad.copy_(w)
            ds.ds_row_renorm([ds.WSeg(w=wpad)], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(wbuf, rows, cols, ld, gu.CANARY_F32), cols
            gu.check_renorm(seg, wpad, eps, what=f"renorm cols={cols}")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_ragged_activation_rows_with_guards(path):
    rng = np.random.default_rng(22)
    eps = 1e-6
    with ds.force_path(path):
        for cols in RAGGED_COLS:
            rows = 19
            ld = ((cols + 7) // 8) * 8 + 16
            act = wl.ActRows("a", wl.normal_bf16(rng, (rows, cols)), wl.normal_bf16(rng, (rows, cols)),
                             wl.alpha_vec(rng, cols))
            xs, rs = [], []
            for src, lst in ((act.x, xs), (act.r, rs)):
                v, b = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
                v.copy_(gu.dev_bf16(src))
                lst.append(v)
            y, ybuf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
            ds.ds_l2_rows([ds.ASeg(x=xs[0], r=rs[0], y=y)], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(ybuf, rows, cols, ld, gu.CANARY_BF16), cols
            gu.check_l2(act, y, eps, what=f"l2 cols={cols}")
            h, hbuf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
            # alpha's storage continues with NaN past cols: none of it may reach a row
            abuf = torch.full((cols + 8,), float("nan"), dtype=torch.float32, device="cuda")
            abuf[:cols].copy_(gu.dev_f32(act.alpha))
            ds.ds_slerp_rows([ds.ASeg(x=xs[0], r=rs[0], y=h, alpha=abuf[:cols])], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(hbuf, rows, cols, ld, gu.CANARY_BF16), cols
            gu.check_slerp(act, h, eps, what=f"slerp cols={cols}")


def test_empty_segments_mixed_in():
    rng = np.random.default_rng(23)
    eps = 1e-6
    segs = [wl.WeightSeg("a", wl.drifted_rows(rng, 5, 64, 1.0), wl.gains(rng, 5), wl.normal_bf16(rng, (5, 64))),
            wl.WeightSeg("empty", np.zeros((0, 64), np.float32), np.zeros(0, np.float32),
                         np.zeros((0, 64), np.uint16)),
            wl.WeightSeg("b", wl.drifted_rows(rng, 300, 96, 1.0), wl.gains(rng, 300),
                         wl.normal_bf16(rng, (300, 96)))]
    outs = gu.run_forward(segs, "f32", eps)
    for s, o in zip(segs, outs):
        if s.rows:
            gu.check_forward(s, o, eps, "f32")
    before = ds.ds_launch_count()
    ds.ds_wn_forward([], "bf16", eps)
    assert ds.ds_launch_count() == before


@pytest.mark.parametrize("path", [ds.DS_PATH_AUTO, ds.DS_PATH_CLUSTER, ds.DS_PATH_TWO_PASS],
                         ids=["auto", "cluster", "two_pass"])
def test_exact_aliasing_allowed(path):
    rng = np.random.default_rng(24)
    act = wl.ActRows("a", wl.normal_bf16(rng, (64, 1000)), wl.normal_bf16(rng, (64, 1000)), wl.alpha_vec(rng, 1000))
    with ds.force_path(path):
        _aliasing(act)


def _aliasing(act):
    (ref,) = gu.run_l2([act], 1e-6)
    (href,) = gu.run_slerp([act], 1e-6)
    for alias in ("x", "r"):
        x, r = gu.dev_bf16(act.x), gu.dev_bf16(act.r)
        ds.ds_l2_rows([ds.ASeg(x=x, r=r, y=x if alias == "x" else r)], 1e-6)
        torch.cuda.synchronize()
        assert torch.equal((x if alias == "x" else r).view(torch.int16), ref.view(torch.int16))
        x, r = gu.dev_bf16(act.x), gu.dev_bf16(act.r)
        ds.ds_slerp_rows([ds.ASeg(x=x, r=r, y=x if alias == "x" else r, alpha=gu.dev_f32(act.alpha))], 1e-6)
        torch.cuda.synchronize()
        assert torch.equal((x if alias == "x" else r).view(torch.int16), href.view(torch.int16))
