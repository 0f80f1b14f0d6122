"""GPU invariants that hold bit for bit, degenerate inputs, negative
controls, and the bounded-wait error path.

* A row's bits never depend on the row count or the segment table
  (TensorFold PR #1260: "a row's bits never depend on the row count").
* Power-of-two scaling of a row leaves its output unchanged at eps = 0 (the
  free scale direction of DragonScale's "Why scales drift"), also through the
  overflow/underflow rescaling path.
* l2 with an all-zero residual equals l2 without one; slerp with alpha = 0
  equals l2 of bf16(l2(res)) (the lerp's multiply-add adds an exact zero);
  at |alpha| = 1 the GPU's b - a may round in fp32, so that end is checked
  against the oracle (where t = b exactly).
* Controls: oracle variants that drop one rounding point must fail the check.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests import gpu_util as gu
from tests.checks import SPREAD, bf16_interval_violations

pytestmark = pytest.mark.gpu

PATHS = [ds.DS_PATH_AUTO, ds.DS_PATH_CTA, ds.DS_PATH_CLUSTER, ds.DS_PATH_TWO_PASS]
PATH_IDS = ["auto", "cta", "cluster", "two_pass"]


def bits(t):
    return t.view(torch.int16)


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_row_count_invariance(path):
    rng = np.random.default_rng(31)
    eps = 1e-6
    with ds.force_path(path):
        for cols in (768, 2048, 4096):
            w = gu.dev_f32(wl.drifted_rows(rng, 97, cols, 0.02))
            g = gu.dev_f32(wl.gains(rng, 97))
            full = torch.empty(97, cols, dtype=torch.bfloat16, device="cuda")
            ds.ds_wn_forward([ds.WSeg(w=w, gain=g, w_eff=full)], "bf16", eps)
            # each row alone, and rows split over many segments in one call
            for r in (0, 41, 96):
                one = torch.empty(1, cols, dtype=torch.bfloat16, device="cuda")
                ds.ds_wn_forward([ds.WSeg(w=w[r:r + 1], gain=g[r:r + 1], w_eff=one)], "bf16", eps)
                assert torch.equal(bits(one[0]), bits(full[r]))
            parts = torch.empty_like(full)
            cuts = [0, 1, 2, 9, 40, 41, 77, 97]
            segs = [ds.WSeg(w=w[a:b], gain=g[a:b], w_eff=parts[a:b]) for a, b in zip(cuts, cuts[1:])]
            ds.ds_wn_forward(segs, "bf16", eps)
            torch.cuda.synchronize()
            assert torch.equal(bits(parts), bits(full))
            x = gu.dev_bf16(wl.normal_bf16(rng, (97, cols)))
            y = torch.empty_like(x)
            ds.ds_l2_rows([ds.ASeg(x=x, y=y)], eps)
            y2 = torch.empty_like(x)
            ds.ds_l2_rows([ds.ASeg(x=x[a:b], y=y2[a:b]) for a, b in zip(cuts, cuts[1:])], eps)
            torch.cuda.synchronize()
            assert torch.equal(bits(y), bits(y2))


def test_whole_model_rows_match_single_segment_calls():
    wk = wl.whole_model(0, n_layer=2, vocab=1000)
    outs = gu.run_forward(wk.weights, "bf16", wk.eps)
    grads = gu.run_backward(wk.weights, "bf16", wk.eps)
    for s, o, (gw, gg) in zip(wk.weights, outs, grads):
        (o1,) = gu.run_forward([s], "bf16", wk.eps)
        assert torch.equal(bits(o), bits(o1)), s.name
        (gw1, gg1), = gu.run_backward([s], "bf16", wk.eps)
        assert torch.equal(gw, gw1) and torch.equal(gg, gg1), s.name


def test_repeat_runs_identical():
    a = wl.activations(3, rows=1024, cols=4096).acts[0]
    h1 = gu.run_slerp([a], 1e-6)[0]
    h2 = gu.run_slerp([a], 1e-6)[0]
    assert torch.equal(bits(h1), bits(h2))
    s = wl.mlp_pair(3).weights[1]
    g1 = gu.run_backward([s], "bf16", 1e-6)[0]
    g2 = gu.run_backward([s], "bf16", 1e-6)[0]
    assert torch.equal(g1[0], g2[0]) and torch.equal(g1[1], g2[1])


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_zero_residual_is_no_residual(path):
    a = wl.activations(4, rows=256, cols=4096).acts[0]
    x = gu.dev_bf16(a.x)
    with ds.force_path(path):
        y0 = torch.empty_like(x)
        ds.ds_l2_rows([ds.ASeg(x=x, y=y0)], 1e-6)
        y1 = torch.empty_like(x)
        ds.ds_l2_rows([ds.ASeg(x=x, r=torch.zeros_like(x), y=y1)], 1e-6)
        torch.cuda.synchronize()
    assert torch.equal(bits(y0), bits(y1))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_slerp_endpoints(path):
    a = wl.activations(5, rows=128, cols=4096).acts[0]
    x, o = gu.dev_bf16(a.x), gu.dev_bf16(a.r)
    C = a.cols
    with ds.force_path(path):
        def l2(t):
            y = torch.empty_like(t)
            ds.ds_l2_rows([ds.ASeg(x=t, y=y)], 1e-6)
            return y

        def slerp(alpha):
            h = torch.empty_like(x)
            ds.ds_slerp_rows([ds.ASeg(x=x, r=o, y=h, alpha=alpha)], 1e-6)
            return h

        h0 = slerp(torch.zeros(C, device="cuda"))
        sign = torch.where(torch.arange(C, device="cuda") % 2 == 0, 1.0, -1.0)
        h1 = slerp(sign)
        ref0 = l2(l2(x))
        torch.cuda.synchronize()
    assert torch.equal(bits(h0), bits(ref0))
    ends = wl.ActRows("a", a.x, a.r, sign.cpu().numpy().astype(np.float32))
    gu.check_slerp(ends, h1, 1e-6, what="slerp |alpha| = 1")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_power_of_two_scale_invariance_eps0(path):
    """W_eff(2^k w) == W_eff(w) and l2(2^k x) == l2(x) bit for bit at eps = 0,
    including k that overflow (k = 60, 70) or underflow (k = -70, -100) the
    fp32 sum of squares and so take the rescaling path."""
    rng = np.random.default_rng(6)
    w = wl.drifted_rows(rng, 16, 4096, 1.0)
    x = wl.normal_bf16(rng, (16, 4096))
    xf = wl.bf16_bits_to_f32(x)
    with ds.force_path(path):
        base = gu.run_forward([wl.WeightSeg("w", w, None, None)], "f32", 0.0)[0]
        ybase = gu.run_l2([wl.ActRows("x", x, None)], 0.0)[0]
        for k in (-100, -70, -20, 20, 60, 70):
            ws = np.ldexp(w, k).astype(np.float32)
            assert np.all(np.isfinite(ws)) and np.array_equal(np.ldexp(ws, -k), w)
            got = gu.run_forward([wl.WeightSeg("w", ws, None, None)], "f32", 0.0)[0]
            assert torch.equal(got, base), k
            xs = wl.to_bf16_bits(np.ldexp(xf, k).astype(np.float32))
            if np.array_equal(wl.bf16_bits_to_f32(xs), np.ldexp(xf, k).astype(np.float32)):
                y = gu.run_l2([wl.ActRows("x", xs, None)], 0.0)[0]
                assert torch.equal(bits(y), bits(ybase)), k


def test_extreme_magnitudes_match_oracle():
    """Rows whose fp32 sum of squares overflows (|x| ~ 1e30) or, at eps = 0,
    underflows (|x| ~ 1e-30, and rows of fp32 subnormals ~ 1e-42) still match
    the float64 oracle.  (The backward of a subnormal row overflows fp32
    legitimately -- 1/n > FLT_MAX -- so it is checked at 1e-30 and above.)"""
    rng = np.random.default_rng(7)
    for scale, eps in ((1e30, 1e-6), (3e37, 0.0), (1e-30, 0.0), (1e-42, 0.0)):
        x = wl.to_bf16_bits((rng.standard_normal((8, 1000)) * scale).astype(np.float32))
        a = wl.ActRows("x", x, None)
        (y,) = gu.run_l2([a], eps, residual=False)
        gu.check_l2(a, y, eps, residual=False, what=f"l2 scale={scale}")
        w = (rng.standard_normal((8, 1000)) * scale).astype(np.float32)
        s = wl.WeightSeg("w", w, wl.gains(rng, 8), rng.standard_normal((8, 1000)).astype(np.float32))
        (o,) = gu.run_forward([s], "f32", eps)
        gu.check_forward(s, o, eps, "f32", what=f"forward scale={scale}")
        if scale >= 1e-30:
            (gw, gg), = gu.run_backward([s], "f32", eps)
            gu.check_backward(s, gw, gg, eps, what=f"backward scale={scale}")


def test_degenerate_rows():
    """Zero rows (eps > 0 -> zeros; eps = 0 -> NaN as 0/0), inf and NaN entries."""
    x = np.zeros((4, 64), np.float32)
    x[1, 3] = np.inf
    x[2, 5] = np.nan
    x[3, :] = 1.0
    a = wl.ActRows("x", wl.to_bf16_bits(x), None)
    for eps in (1e-6, 0.0):
        (y,) = gu.run_l2([a], eps, residual=False)
        gu.check_l2(a, y, eps, residual=False, what=f"degenerate eps={eps}")
        s = wl.WeightSeg("w", x.copy(), None, np.ones_like(x))
        (o,) = gu.run_forward([s], "f32", eps)
        gu.check_forward(s, o, eps, "f32", what=f"degenerate forward eps={eps}")


def test_integer_rows_exact_sums():
    """Integer rows: every fp32 partial sum is exact (< 2^24), far above fp16's
    range; only the square root, division and product round."""
    x = wl.integer_rows(8, 64, 4096)
    a = wl.ActRows("x", x, wl.integer_rows(9, 64, 4096))
    for res in (False, True):
        (y,) = gu.run_l2([a], 1e-6, residual=res)
        gu.check_l2(a, y, 1e-6, residual=res, what="integer rows")


# ------------------------------------------------------------ negative controls

def test_controls_fail_against_the_gpu():
    a = wl.activations(0, rows=256, cols=4096).acts[0]
    (y,) = gu.run_l2([a], 1e-6, residual=True)
    gy = gu.host_bits(y)
    lo, hi = oracle.l2_rows_interval(a.x, a.r, delta=SPREAD, flags=oracle.OR_DROP_SUM_ROUND)
    assert bf16_interval_violations(gy, lo, hi).any(axis=1).any(), "dropping bf16(x + r) went unnoticed"
    (h,) = gu.run_slerp([a], 1e-6)
    gh = gu.host_bits(h)
    for f in (oracle.OR_DROP_SLERP_A, oracle.OR_DROP_SLERP_B):
        lo, hi = oracle.slerp_rows_interval(a.x, a.r, a.alpha, delta=SPREAD, flags=f)
        assert bf16_interval_violations(gh, lo, hi).any(axis=1).any(), f
    small = wl.ActRows("s", wl.small_norm_rows(5, 64, 4096), None)
    (ys,) = gu.run_l2([small], 1e-6, residual=False)
    gys = gu.host_bits(ys)
    for f in (oracle.OR_EPS_OUTSIDE, oracle.OR_EPS_ZERO):
        lo, hi = oracle.l2_rows_interval(small.x, None, delta=SPREAD, flags=f)
        assert bf16_interval_violations(gys, lo, hi).any(axis=1).any(), f
    # and the definition itself passes on the same outputs
    gu.check_l2(a, y, 1e-6)
    gu.check_slerp(a, h, 1e-6)
    gu.check_l2(small, ys, 1e-6, residual=False)


# ------------------------------------------------------------- error paths ---

def test_bounded_wait_reports_timeout():
    assert ds.ds_get_device_status() == ds.DS_OK
    ds.ds_debug_wait_timeout_selftest(2_000_000)  # 2 ms; nothing ever arrives
    assert ds.ds_get_device_status() == ds.DS_ERR_DEVICE_TIMEOUT
    assert ds.ds_get_device_status() == ds.DS_OK   # read clears it
    # the context is still usable
    a = wl.tiny(0).acts[0]
    (y,) = gu.run_l2([a], 1e-6)
    gu.check_l2(a, y, 1e-6)


def test_launch_counter_counts_kernels():
    wk = wl.whole_model(0, n_layer=1, vocab=512)
    before = ds.ds_launch_count()
    gu.run_forward(wk.weights, "bf16", wk.eps)
    assert ds.ds_launch_count() - before == 1   # every staged row width in one launch
