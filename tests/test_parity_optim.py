"""GPU parity of the optimizer companions of method "rescale" (DragonScale
package description, "Optimizer"): ds_grad_project and ds_renorm_momentum
against the float64 oracle on the same seeded inputs, on every row class,
with ragged and padded shapes, the config shapes and the rescale path."""
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


def _state(weights, seed=0):
    return wl.with_fp32_state(weights, seed)


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_tiny_all_paths(path, eps):
    seg = _state(wl.tiny(0).weights)[0]
    emb = wl.WeightSeg("emb", seg.w, None, seg.gy, radius=float(np.sqrt(seg.cols)))
    with ds.force_path(path):
        (G,) = gu.run_project([seg], eps)
        gu.check_project(seg, G, eps)
        for s in (seg, emb):
            ((w, m),) = gu.run_momentum([s], eps)
            gu.check_momentum(s, w, m, eps)


RAGGED_COLS = [1, 3, 5, 7, 8, 13, 127, 129, 255, 257, 1000, 1023, 2047, 2049, 4097]


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_ragged_rows_with_guards(path):
    rng = np.random.default_rng(41)
    eps = 1e-6
    with ds.force_path(path):
        for cols in RAGGED_COLS:
            rows = 23
            ld = ((cols + 3) // 4) * 4 + 4
            seg = wl.WeightSeg("r", wl.drifted_rows(rng, rows, cols, 0.5), None,
                               rng.standard_normal((rows, cols), dtype=np.float32))
            w, wbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            w.copy_(gu.dev_f32(seg.w))
            G, gbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            G.copy_(gu.dev_f32(seg.gy))
            ds.ds_grad_project([ds.WSeg(w=w, grad_w=G)], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(gbuf, rows, cols, ld, gu.CANARY_F32), cols
            assert gu.guards_intact(wbuf, rows, cols, ld, gu.CANARY_F32), cols
            assert torch.equal(w, gu.dev_f32(seg.w))                  # w is read-only here
            gu.check_project(seg, G, eps, what=f"grad_project cols={cols}")
            m, mbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
            m.copy_(gu.dev_f32(seg.gy))
            ds.ds_renorm_momentum([ds.WSeg(w=w, grad_w=m)], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(mbuf, rows, cols, ld, gu.CANARY_F32), cols
            assert gu.guards_intact(wbuf, rows, cols, ld, gu.CANARY_F32), cols
            gu.check_momentum(seg, w, m, eps, what=f"renorm_momentum cols={cols}")


def test_mlp_pair_one_call():
    segs = _state(wl.mlp_pair(0).weights, 1)
    before = ds.ds_launch_count()
    Gs = gu.run_project(segs, 1e-6)
    assert ds.ds_launch_count() - before == 1
    for s, G in zip(segs, Gs):
        gu.check_project(s, G, 1e-6, what=f"{s.name} grad_project")
    for s, (w, m) in zip(segs, gu.run_momentum(segs, 1e-6)):
        gu.check_momentum(s, w, m, 1e-6, what=f"{s.name} renorm_momentum")


def test_whole_model_one_call():
    segs = _state(wl.whole_model(0).weights, 2)
    before = ds.ds_launch_count()
    Gs = gu.run_project(segs, 1e-6)
    assert ds.ds_launch_count() - before == 1
    res = gu.run_momentum(segs, 1e-6)
    for i, (s, G, (w, m)) in enumerate(zip(segs, Gs, res)):
        rows = gu.sample_rows(s.rows, 6 if s.rows < 30000 else 64, 200 + i)
        gu.check_project(s, G, 1e-6, rows=rows, what=f"{s.name} grad_project")
        gu.check_momentum(s, w, m, 1e-6, rows=rows, what=f"{s.name} renorm_momentum")


def test_wide_and_long_rows():
    wk = wl.wide(0)
    lr = wl.long_rows(0)
    segs = _state(wk.weights + lr.weights, 3)
    Gs = gu.run_project(segs, 1e-6)
    res = gu.run_momentum(segs, 1e-6)
    for i, (s, G, (w, m)) in enumerate(zip(segs, Gs, res)):
        rows = gu.sample_rows(s.rows, min(s.rows, 24), 300 + i)
        gu.check_project(s, G, 1e-6, rows=rows, what=f"{s.name} grad_project")
        gu.check_momentum(s, w, m, 1e-6, rows=rows, what=f"{s.name} renorm_momentum")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_pow2_scale_invariance_eps0(path):
    """At eps = 0 only the row's direction matters: w scaled by 2^k (exact in
    fp32) gives the same projected gradient and the same renormed row, bit
    for bit, on both sides of the power-of-two rescale."""
    rng = np.random.default_rng(43)
    w = wl.drifted_rows(rng, 16, 300, 1.0)
    G = rng.standard_normal(w.shape, dtype=np.float32)
    seg = wl.WeightSeg("s", w, None, G)
    with ds.force_path(path):
        (G0,) = gu.run_project([seg], 0.0)
        ((w0, m0),) = gu.run_momentum([seg], 0.0)
        for k in (-100, -70, -20, 20, 60, 70):
            sk = wl.WeightSeg("s", np.ldexp(w, k).astype(np.float32), None, G)
            assert np.all(np.isfinite(sk.w)) and np.all(sk.w[w != 0] != 0)
            (Gk,) = gu.run_project([sk], 0.0)
            ((wk, mk),) = gu.run_momentum([sk], 0.0)
            assert torch.equal(Gk, G0), k
            assert torch.equal(mk, m0), k
            assert torch.equal(wk, w0), k
        gu.check_project(seg, G0, 0.0)


def test_extreme_magnitudes():
    """Rows whose fp32 sum of squares overflows (|w| ~ 1e30, 3e37) or, at
    eps = 0, underflows (|w| ~ 1e-30, and rows of fp32 subnormals ~ 1e-42)
    go through the exact power-of-two rescale and still match the f64
    definition (the projection and the renormed row stay finite there)."""
    rng = np.random.default_rng(44)
    for scale, eps in ((1e30, 1e-6), (3e37, 0.0), (1e-30, 0.0), (1e-42, 0.0)):
        w = (rng.standard_normal((8, 1000)) * scale).astype(np.float32)
        G = rng.standard_normal((8, 1000)).astype(np.float32)
        seg = wl.WeightSeg("x", w, None, G)
        for path in PATHS:
            with ds.force_path(path):
                (Gp,) = gu.run_project([seg], eps)
                gu.check_project(seg, Gp, eps, what=f"scale={scale} path={path}")
                ((wo, mo),) = gu.run_momentum([seg], eps)
                gu.check_momentum(seg, wo, mo, eps, what=f"scale={scale} path={path}")


def test_zero_rows_and_determinism():
    rng = np.random.default_rng(45)
    w = wl.drifted_rows(rng, 40, 640, 1.0)
    w[[3, 17]] = 0.0
    G = rng.standard_normal(w.shape, dtype=np.float32)
    seg = wl.WeightSeg("z", w, None, G)
    (Ga,) = gu.run_project([seg], 1e-6)
    (Gb,) = gu.run_project([seg], 1e-6)
    assert torch.equal(Ga, Gb)
    h = gu.host_f32(Ga)
    assert np.array_equal(h[[3, 17]], G[[3, 17]])            # nothing to remove from a zero row
    ((wo, mo),) = gu.run_momentum([seg], 1e-6)
    assert not gu.host_f32(wo)[[3, 17]].any()
    gu.check_momentum(seg, wo, mo, 1e-6)


def test_eps_control_is_detected():
    """A planted mistake on the oracle side (eps dropped) must fail the
    comparison on small-norm rows: the check is sharp enough to see eps."""
    rng = np.random.default_rng(46)
    w = (wl.drifted_rows(rng, 32, 256, 1.0) * np.float32(2e-4)).astype(np.float32)
    G = rng.standard_normal(w.shape, dtype=np.float32)
    seg = wl.WeightSeg("c", w, None, G)
    (Gp,) = gu.run_project([seg], 1e-6)
    gu.check_project(seg, Gp, 1e-6)
    import oracle

    with pytest.raises(AssertionError):
        gu.check_project(seg, Gp, 1e-6, flags=oracle.OR_EPS_ZERO)


def test_largest_weight_slot_ragged_with_guards():
    """Rows of 12,289 fp32 columns: 96 KB of staged input in the widest
    layout, so the 112 KB-slot class (two positions, eight warps per row),
    with a ragged last quad and padded rows."""
    rng = np.random.default_rng(47)
    rows, cols = 9, 12289
    assert ds.ds_row_class(ds.DS_OP_WN_BACKWARD, cols)[:2] == (ds.DS_PATH_CTA, 256)
    ld = ((cols + 3) // 4) * 4 + 4
    seg = wl.WeightSeg("big", wl.drifted_rows(rng, rows, cols, 0.02), wl.gains(rng, rows),
                       rng.standard_normal((rows, cols), dtype=np.float32))
    w, wbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
    w.copy_(gu.dev_f32(seg.w))
    g = gu.dev_f32(seg.g)
    gy, _ = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
    gy.copy_(gu.dev_f32(seg.gy))
    gw, gwbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
    gg = torch.empty(rows, device="cuda")
    ds.ds_wn_backward([ds.WSeg(w=w, gain=g, gy=gy, grad_w=gw, grad_g=gg)], "f32", 1e-6)
    torch.cuda.synchronize()
    assert gu.guards_intact(gwbuf, rows, cols, ld, gu.CANARY_F32)
    gu.check_backward(seg, gw, gg, 1e-6, what="backward 112 KB slots")
    G, gbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
    G.copy_(gu.dev_f32(seg.gy))
    ds.ds_grad_project([ds.WSeg(w=w, grad_w=G)], 1e-6)
    torch.cuda.synchronize()
    assert gu.guards_intact(gbuf, rows, cols, ld, gu.CANARY_F32)
    gu.check_project(seg, G, 1e-6, what="grad_project 112 KB slots")
    m, mbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
    m.copy_(gu.dev_f32(seg.gy))
    ds.ds_renorm_momentum([ds.WSeg(w=w, grad_w=m)], 1e-6)
    torch.cuda.synchronize()
    assert gu.guards_intact(mbuf, rows, cols, ld, gu.CANARY_F32)
    assert gu.guards_intact(wbuf, rows, cols, ld, gu.CANARY_F32)
    gu.check_momentum(seg, w, m, 1e-6, what="renorm_momentum 112 KB slots")
