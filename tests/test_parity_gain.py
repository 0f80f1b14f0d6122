"""GPU parity of the row lengths, the preserving gain and the scalar gain
(DragonScale package description: options table -- `gain` "scalar", `init`
"preserve" -- and "Monitor": each layer's raw row lengths) against the
float64 oracle, on every row class the weight calls use."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests import gpu_util as gu
from tests.checks import rel_violations

pytestmark = pytest.mark.gpu

PATHS = [ds.DS_PATH_AUTO, ds.DS_PATH_WARP, ds.DS_PATH_CTA, ds.DS_PATH_CLUSTER, ds.DS_PATH_TWO_PASS]
PATH_IDS = ["auto", "warp", "cta", "cluster", "two_pass"]


def run_norms(w: np.ndarray, eps: float, preserve=False, radius=1.0, ld_pad=0):
    R, C = w.shape
    ld = (C + 3) // 4 * 4 + ld_pad         # rows start on 16 bytes
    wd, _ = gu.padded(R, C, ld, torch.float32, gu.CANARY_F32)
    wd.copy_(gu.dev_f32(w))
    out = torch.full((R + 1,), -1.0, dtype=torch.float32, device="cuda")
    seg = ds.WSeg(w=wd, rnorm=out[:R], radius=radius)
    (ds.ds_gain_preserve if preserve else ds.ds_row_norms)([seg], eps)
    torch.cuda.synchronize()
    h = gu.host_f32(out)
    assert h[R] == -1.0          # nothing past the rows
    return h[:R]


@pytest.mark.parametrize("eps", [1e-6, 0.0])
@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_row_norms_shapes(eps, path):
    """Every row class: the staged kernel (a row per warp, per CTA or split
    over a cluster) and the warp-per-row kernel for rows past the staged
    classes (forced here with the two-pass path)."""
    rng = np.random.default_rng(81)
    with ds.force_path(path):
        for R, C in ((1, 1), (7, 3), (33, 129), (64, 768), (5, 4097), (3, 131072), (300, 2048), (9, 40000)):
            w = wl.drifted_rows(rng, R, C, 0.02)
            got = run_norms(w, eps, ld_pad=4)
            ref = oracle.row_norms(w, eps=eps)
            bad = rel_violations(got, ref, 2e-6)
            assert not bad.any(), (R, C, got[bad][:3], ref[bad][:3])


@pytest.mark.parametrize("path", [ds.DS_PATH_AUTO, ds.DS_PATH_TWO_PASS], ids=["staged", "warp_per_row"])
def test_row_norms_whole_model(path):
    """The whole-model table (85 segments) in one call, every row against
    the oracle; the staged kernel takes it in one launch."""
    wk = wl.whole_model(0)
    outs, segs = [], []
    for s in wk.weights:
        wd = gu.dev_f32(s.w)
        out = torch.full((s.rows,), -1.0, dtype=torch.float32, device="cuda")
        outs.append((s, out, wd))
        segs.append(ds.WSeg(w=wd, rnorm=out))
    with ds.force_path(path):
        before = ds.ds_launch_count()
        ds.ds_row_norms(segs, 1e-6)
        torch.cuda.synchronize()
        launches = ds.ds_launch_count() - before
    if path == ds.DS_PATH_AUTO:
        assert launches == 1, launches
    for s, out, _ in outs:
        ref = oracle.row_norms(s.w, eps=1e-6)
        bad = rel_violations(gu.host_f32(out), ref, 2e-6)
        assert not bad.any(), (s.name, int(bad.sum()))


def test_row_norms_extreme_and_zero_rows():
    rng = np.random.default_rng(82)
    for scale, eps in ((1e30, 1e-6), (3e37, 0.0), (1e-30, 0.0), (1e-42, 0.0)):
        w = (rng.standard_normal((6, 1000)) * scale).astype(np.float32)
        got = run_norms(w, eps)
        ref = oracle.row_norms(w, eps=eps)
        fin = ref < float(np.finfo(np.float32).max)
        # 2e-6 relative, or one step of fp32's subnormal spacing for lengths below 2^-126
        err = np.abs(got[fin].astype(np.float64) - ref[fin])
        assert np.all(err <= np.maximum(2e-6 * ref[fin], 2.0 ** -149)), scale
        assert np.all(np.isinf(got[~fin]))   # lengths past fp32's range are inf
    w = np.zeros((3, 64), np.float32)
    assert np.all(run_norms(w, 1e-6) == np.float32(np.sqrt(np.float32(1e-6))))
    assert np.all(run_norms(w, 0.0) == 0.0)


def test_preserving_gain_keeps_the_output():
    rng = np.random.default_rng(83)
    w = wl.drifted_rows(rng, 40, 768, 0.02)
    for radius in (1.0, float(np.sqrt(768))):
        g = run_norms(w, 1e-6, preserve=True, radius=radius)
        ref = oracle.row_norms(w, eps=1e-6, div=radius)
        assert not rel_violations(g, ref, 2e-6).any()
        seg = wl.WeightSeg("p", w, g, None, radius=radius)
        (weff,) = gu.run_forward([seg], "f32", 1e-6)
        got = gu.host_f32(weff)
        assert not rel_violations(got, w.astype(np.float64), 4e-7).any()


def _scalar_and_channel(seg, g: float, path, gy_dtype="bf16"):
    """GPU backward of seg with one scalar gain g, and with a per-row gain
    array of g: returns (grad_w, grad_g [R + 1]) and (grad_w, grad_g [R])."""
    R, C = seg.w.shape
    with ds.force_path(path):
        w = gu.dev_f32(seg.w)
        gy = gu.dev_bf16(seg.gy) if gy_dtype == "bf16" else gu.dev_f32(seg.gy)
        gs = torch.full((1,), g, dtype=torch.float32, device="cuda")
        gw_s = torch.empty_like(w)
        gg_s = torch.empty(R + 1, dtype=torch.float32, device="cuda")
        ds.ds_wn_backward([ds.WSeg(w=w, gain=gs, gy=gy, grad_w=gw_s, grad_g=gg_s, radius=seg.radius,
                                   gain_scalar=True)], gy_dtype, 1e-6)
        gc = torch.full((R,), g, dtype=torch.float32, device="cuda")
        gw_c = torch.empty_like(w)
        gg_c = torch.empty(R, dtype=torch.float32, device="cuda")
        ds.ds_wn_backward([ds.WSeg(w=w, gain=gc, gy=gy, grad_w=gw_c, grad_g=gg_c, radius=seg.radius)],
                          gy_dtype, 1e-6)
        # forward: the scalar gain and the array of it give the same bits
        o_s = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
        o_c = torch.empty_like(o_s)
        ds.ds_wn_forward([ds.WSeg(w=w, gain=gs, w_eff=o_s, radius=seg.radius, gain_scalar=True)], "bf16", 1e-6)
        ds.ds_wn_forward([ds.WSeg(w=w, gain=gc, w_eff=o_c, radius=seg.radius)], "bf16", 1e-6)
        torch.cuda.synchronize()
        assert torch.equal(o_s, o_c)
    return (gw_s, gu.host_f32(gg_s)), (gw_c, gu.host_f32(gg_c))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_scalar_gain_matches_channel_and_oracle(path):
    rng = np.random.default_rng(84)
    R, C = 300, 1000
    w = wl.drifted_rows(rng, R, C, 0.02)
    gy = wl.normal_bf16(rng, (R, C), 1e-3)
    seg = wl.WeightSeg("s", w, None, gy, radius=1.0)
    g = 1.75
    (gw_s, gg_s), (gw_c, gg_c) = _scalar_and_channel(seg, g, path)
    assert torch.equal(gw_s, gw_c)                        # grad_w: the same arithmetic
    assert np.array_equal(gg_s[:R], gg_c)                 # the per-row parts
    assert abs(float(gg_s[R]) - float(np.sum(gg_s[:R], dtype=np.float64))) <= \
        np.spacing(np.float32(abs(gg_s[R])))              # their sum, rounded once
    ref_w, parts, tot = oracle.wn_backward_scalar_gain(w, gy, g, eps=1e-6, nthreads=oracle.default_threads())
    gy64 = wl.bf16_bits_to_f32(gy).astype(np.float64)
    floor = np.linalg.norm(gy64, axis=1)
    assert not rel_violations(gg_s[:R], parts, 1e-5, floor).any()
    assert abs(gg_s[R] - tot) <= 1e-5 * floor.sum()


def test_scalar_gain_whole_model_one_call():
    segs = wl.whole_model(0).weights[:12]
    cs, outs = [], []
    for s in segs:
        R = s.rows
        w = gu.dev_f32(s.w)
        gs = torch.full((1,), 0.5, dtype=torch.float32, device="cuda")
        gw = torch.empty_like(w)
        gg = torch.empty(R + 1, dtype=torch.float32, device="cuda")
        cs.append(ds.WSeg(w=w, gain=gs, gy=gu.dev_bf16(s.gy), grad_w=gw, grad_g=gg, radius=s.radius,
                          gain_scalar=True))
        outs.append(gg)
    ds.ds_wn_backward(cs, "bf16", 1e-6)
    torch.cuda.synchronize()
    for s, gg in zip(segs, outs):
        h = gu.host_f32(gg)
        _, parts, tot = oracle.wn_backward_scalar_gain(s.w, s.gy, 0.5, rho=s.radius, eps=1e-6,
                                                       nthreads=oracle.default_threads())
        floor = s.radius * np.linalg.norm(wl.bf16_bits_to_f32(s.gy).astype(np.float64), axis=1)
        assert abs(h[s.rows] - tot) <= 1e-5 * floor.sum(), s.name
