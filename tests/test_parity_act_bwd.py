"""GPU parity of the activation backward calls (ds_l2_rows_backward,
ds_slerp_rows_backward) against the float64 oracle on the same inputs.

Tolerances (fp32 gradients, like grad_w): |gpu - ref| <= 1e-5 * max(|ref|,
floor) with a floor of the row's gradient scale (the projections' subtraction
can cancel).  The l2 backward's one rounding point, s = bf16(x + r), is taken
identically on both sides, so it is checked at that bound everywhere.  slerp
rounds a = bf16(res/na) and b = bf16(out/nb): where the f64 quotient lies
within the GPU's fp32 spread of a bf16 halfway point, either rounding is the
forward's value, and one bf16 step of a_j or b_j moves t_j, dt_j and the row's
dalpha part at that column by about 2^-8 of their size.  So: exactly
representable rows (+-1 entries, 4^k columns, eps = 0, where a and b are
exact) are checked at 1e-5 everywhere, dalpha included.  Random rows are
checked at 1e-5 plus the bounded effect of each flagged rounding: on its row
through the row's sum of squares (a common factor 1/nt) and t . dh, and at
the flagged column through its own dt_j; dalpha per column likewise.
"""
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

PATHS = [ds.DS_PATH_AUTO, ds.DS_PATH_WARP, ds.DS_PATH_CTA]
PATH_IDS = ["auto", "warp", "cta"]


def f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def run_l2_bwd(x, r, dy, eps, ld=None, ld_d=None):
    R, C = x.shape
    xd, dyd = gu.dev_bf16(x), gu.dev_bf16(dy)
    rd = gu.dev_bf16(r) if r is not None else None
    dx = torch.empty(R, C, dtype=torch.float32, device="cuda")
    ds.ds_l2_rows_backward([ds.AGSeg(x=xd, r=rd, dy=dyd, dx=dx)], eps)
    torch.cuda.synchronize()
    return gu.host_f32(dx)


def run_slerp_bwd(res, out, alpha, dh, eps, with_dalpha=True):
    R, C = res.shape
    dres = torch.empty(R, C, dtype=torch.float32, device="cuda")
    dout = torch.empty_like(dres)
    da = torch.empty(C, dtype=torch.float32, device="cuda") if with_dalpha else None
    ds.ds_slerp_rows_backward([ds.AGSeg(x=gu.dev_bf16(res), r=gu.dev_bf16(out), dy=gu.dev_bf16(dh), dx=dres,
                                        dr=dout, alpha=gu.dev_f32(alpha))], eps, dalpha=da)
    torch.cuda.synchronize()
    return gu.host_f32(dres), gu.host_f32(dout), (gu.host_f32(da) if with_dalpha else None)


def check_l2_bwd(x, r, dy, got, eps, what=""):
    ref = oracle.l2_rows_backward(x, r, dy, eps=eps, nthreads=oracle.default_threads())
    s = f64(x) + (f64(r) if r is not None else 0.0)
    n = np.sqrt((s * s).sum(1) + eps)
    floor = (np.sqrt(np.mean(f64(dy) ** 2, axis=1)) / n)[:, None]
    bad = rel_violations(got, ref, 1e-5, floor)
    assert not bad.any(), f"{what}: {int(bad.sum())} dx entries beyond tolerance (first {np.argwhere(bad)[0]})"


def ambiguous(v, nrm, window=4e-7):
    """Elements whose quotient v / nrm (f64) lies within `window` (relative) of
    a bf16 halfway point: the GPU's fp32 quotient may round either way."""
    q = v / nrm[:, None]
    bits = oracle.bf16_rne_array(q)
    lo = oracle.bf16_rne_array(q * (1 - window))
    hi = oracle.bf16_rne_array(q * (1 + window))
    return (lo != bits) | (hi != bits)


def check_slerp_bwd(res, out, alpha, dh, got, eps, strict, what=""):
    dres, dout, da = got
    nt = oracle.default_threads()
    rr, ro, rda = oracle.slerp_rows_backward(res, out, alpha, dh, eps=eps, nthreads=nt, dalpha=da is not None)
    a64, b64, d64 = f64(res), f64(out), f64(dh)
    na = np.sqrt((a64 * a64).sum(1) + eps)
    nb = np.sqrt((b64 * b64).sum(1) + eps)
    g = np.sqrt(np.mean(d64 ** 2, axis=1))
    # the forward's a, b and t (host arithmetic on the same rounding rule)
    ah = f64(oracle.bf16_rne_array(a64 / na[:, None]))
    bh = f64(oracle.bf16_rne_array(b64 / nb[:, None]))
    t = ah + np.abs(alpha.astype(np.float64)) * (bh - ah)
    St = (t * t).sum(1) + eps
    it = 1.0 / np.sqrt(St)
    Dt = (t * d64).sum(1)
    flag = np.zeros(res.shape, bool) if strict else (ambiguous(a64, na) | ambiguous(b64, nb))
    # A flagged rounding moves t_j by up to dt_j = 2^-7 max(|a_j|, |b_j|): the
    # row's sum of squares by 2 |t_j| dt_j (a common factor on the row through
    # 1/nt) and t . dh by dt_j |dh_j| (through t_k Dt/nt^2); margin 2.
    dtj = np.where(flag, 2.0 ** -7 * np.maximum(np.abs(ah), np.abs(bh)), 0.0)
    dSt = (2 * np.abs(t) * dtj + dtj ** 2).sum(1)
    dDt = (dtj * np.abs(d64)).sum(1)
    rowrel = 2 * dSt / (2 * St)
    rowabs = 2 * np.abs(t) * ((dDt + np.abs(Dt) * dSt / St) / St * it)[:, None]
    # At the flagged column itself the flip also moves dt_j = (dh_j - t_j Dt/nt^2)/nt
    # by dt_j's share of it, |delta t_j| |Dt| / nt^3, and with it da_j, db_j and
    # dres_j, dout_j (divided by na, nb; the factors (1 - |alpha|), |alpha| are
    # at most 1); margin 2 on top of dtj, itself an upper bound of the step.
    local = 2 * dtj * (np.abs(Dt) * it ** 3)[:, None]
    for got_x, ref_x, nrm, name in ((dres, rr, na, "dres"), (dout, ro, nb, "dout")):
        floor = (g / nrm)[:, None]
        allowed = 1e-5 * np.maximum(np.abs(ref_x), floor) + rowrel[:, None] * np.abs(ref_x) + rowabs / nrm[:, None] \
            + local / nrm[:, None]
        diff = np.abs(got_x - ref_x)
        bad = ~(diff <= allowed) & ~(np.isnan(got_x) & np.isnan(ref_x))
        assert not bad.any(), f"{what}: {int(bad.sum())} {name} entries beyond tolerance (first {np.argwhere(bad)[0]}, " \
                              f"flagged {int(flag.sum())})"
    if da is not None:
        # dalpha_j sums the rows' sign(alpha_j) (b_j - a_j) dt_j.  Each part
        # carries fp32 error of order 1e-5 |b_j - a_j| |dh|/nt (dt is a
        # projection that can cancel); flagged roundings move parts locally
        # (2^-6 |dh|/nt) and through the row factors above.
        unit = (g * it)[:, None]
        floor = (np.abs(bh - ah) * unit).sum(0)
        flips = (flag * unit).sum(0) * 2.0 ** -6
        rows_f = (np.abs(bh - ah) * (rowrel[:, None] * unit + rowabs)).sum(0)
        allowed = 1e-5 * np.maximum(np.abs(rda), floor) + flips + rows_f
        bad = np.abs(da - rda) > allowed
        assert not bad.any(), f"{what}: {int(bad.sum())} dalpha entries beyond tolerance (first {np.argwhere(bad)[0]})"


# ------------------------------------------------------------------- l2 ----

@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("residual", [False, True], ids=["plain", "residual"])
def test_l2_backward_tiny(path, residual):
    rng = np.random.default_rng(71)
    x = wl.normal_bf16(rng, (32, 128))
    r = wl.normal_bf16(rng, (32, 128)) if residual else None
    dy = wl.normal_bf16(rng, (32, 128))
    with ds.force_path(path):
        for eps in (1e-6, 0.0):
            got = run_l2_bwd(x, r, dy, eps)
            check_l2_bwd(x, r, dy, got, eps, what=f"l2 bwd eps={eps}")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_l2_backward_ragged_with_guards(path):
    rng = np.random.default_rng(72)
    with ds.force_path(path):
        for cols in (1, 3, 7, 8, 13, 127, 129, 1000, 2049, 4097, 10920):
            rows = 11
            ld = ((cols + 7) // 8) * 8 + 16
            ldd = ((cols + 3) // 4) * 4 + 8
            x, r, dy = (wl.normal_bf16(rng, (rows, cols)) for _ in range(3))
            bufs = []
            for src in (x, r, dy):
                v, _ = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
                v.copy_(gu.dev_bf16(src))
                bufs.append(v)
            dx, dxbuf = gu.padded(rows, cols, ldd, torch.float32, gu.CANARY_F32)
            ds.ds_l2_rows_backward([ds.AGSeg(x=bufs[0], r=bufs[1], dy=bufs[2], dx=dx)], 1e-6)
            torch.cuda.synchronize()
            assert gu.guards_intact(dxbuf, rows, cols, ldd, gu.CANARY_F32), cols
            check_l2_bwd(x, r, dy, gu.host_f32(dx), 1e-6, what=f"l2 bwd cols={cols}")


def test_l2_backward_config_rows_sampled():
    act = wl.activations(0, 16384, 4096).acts[0]
    rows = gu.sample_rows(act.rows, 96, 73)
    rng = np.random.default_rng(74)
    dy = wl.normal_bf16(rng, (act.rows, act.cols))
    for r in (None, act.r):
        got = run_l2_bwd(act.x, r, dy, 1e-6)
        check_l2_bwd(act.x[rows], None if r is None else r[rows], dy[rows], got[rows], 1e-6,
                     what=f"l2 bwd [16384,4096] residual={r is not None}")


def test_l2_backward_extreme_magnitudes():
    """|x| ~ 1e30 (sum of squares overflows fp32) and, at eps = 0, 1e-30
    (underflows): the power-of-two rescale path."""
    rng = np.random.default_rng(75)
    for scale, eps in ((1e30, 1e-6), (3e37, 0.0), (1e-30, 0.0)):
        x = wl.to_bf16_bits((rng.standard_normal((8, 1000)) * scale).astype(np.float32))
        dy = wl.normal_bf16(rng, (8, 1000))
        got = run_l2_bwd(x, None, dy, eps)
        check_l2_bwd(x, None, dy, got, eps, what=f"l2 bwd scale={scale}")


def test_l2_backward_eps_control_detected():
    rng = np.random.default_rng(76)
    x = wl.small_norm_rows(77, 16, 512)
    dy = wl.normal_bf16(rng, (16, 512))
    got = run_l2_bwd(x, None, dy, 1e-6)
    check_l2_bwd(x, None, dy, got, 1e-6)
    ref0 = oracle.l2_rows_backward(x, None, dy, eps=1e-6, flags=oracle.OR_EPS_ZERO)
    assert rel_violations(got, ref0, 1e-5).any()


# ---------------------------------------------------------------- slerp ----

def exact_rows(rng, R, C):
    """+-1 entries: with C = 4^k and eps = 0, res / na = +-2^-k is a bf16 value."""
    return wl.to_bf16_bits(rng.choice([-1.0, 1.0], size=(R, C)).astype(np.float32))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("C", [64, 256, 1024, 4096])
def test_slerp_backward_exact_rows(path, C):
    rng = np.random.default_rng(78 + C)
    R = 40
    res, out = exact_rows(rng, R, C), exact_rows(rng, R, C)
    alpha = wl.alpha_vec(rng, C, std=0.3)
    dh = wl.normal_bf16(rng, (R, C))
    with ds.force_path(path):
        got = run_slerp_bwd(res, out, alpha, dh, 0.0)
    check_slerp_bwd(res, out, alpha, dh, got, 0.0, strict=True, what=f"slerp bwd exact C={C}")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_slerp_backward_tiny(path):
    rng = np.random.default_rng(79)
    res, out, dh = (wl.normal_bf16(rng, (32, 128)) for _ in range(3))
    alpha = wl.alpha_vec(rng, 128)
    with ds.force_path(path):
        got = run_slerp_bwd(res, out, alpha, dh, 1e-6)
    check_slerp_bwd(res, out, alpha, dh, got, 1e-6, strict=False, what="slerp bwd tiny")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_slerp_backward_ragged_with_guards(path):
    rng = np.random.default_rng(80)
    with ds.force_path(path):
        for cols in (1, 5, 8, 13, 129, 1000, 4097, 7168, 10920):
            rows = 9
            ld = ((cols + 7) // 8) * 8 + 8
            ldd = ((cols + 3) // 4) * 4 + 4
            res, out, dh = (wl.normal_bf16(rng, (rows, cols)) for _ in range(3))
            alpha = wl.alpha_vec(rng, cols)
            abuf = torch.full((cols + 8,), float("nan"), dtype=torch.float32, device="cuda")
            abuf[:cols].copy_(gu.dev_f32(alpha))
            ins = []
            for src in (res, out, dh):
                v, _ = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
                v.copy_(gu.dev_bf16(src))
                ins.append(v)
            dres, b1 = gu.padded(rows, cols, ldd, torch.float32, gu.CANARY_F32)
            dout, b2 = gu.padded(rows, cols, ldd, torch.float32, gu.CANARY_F32)
            da = torch.empty(cols, dtype=torch.float32, device="cuda")
            ds.ds_slerp_rows_backward([ds.AGSeg(x=ins[0], r=ins[1], dy=ins[2], dx=dres, dr=dout,
                                                alpha=abuf[:cols])], 1e-6, dalpha=da)
            torch.cuda.synchronize()
            assert gu.guards_intact(b1, rows, cols, ldd, gu.CANARY_F32), cols
            assert gu.guards_intact(b2, rows, cols, ldd, gu.CANARY_F32), cols
            got = (gu.host_f32(dres), gu.host_f32(dout), gu.host_f32(da))
            check_slerp_bwd(res, out, alpha, dh, got, 1e-6, strict=False, what=f"slerp bwd cols={cols}")


def test_slerp_backward_config_shapes():
    """[2048, 4096] of the activation workload (its dalpha over all 2048
    rows) and sampled rows of [8192, 7168] (64 KB slots)."""
    act = wl.activations(0, 2048, 4096).acts[0]
    rng = np.random.default_rng(81)
    dh = wl.normal_bf16(rng, (act.rows, act.cols))
    got = run_slerp_bwd(act.x, act.r, act.alpha, dh, 1e-6)
    check_slerp_bwd(act.x, act.r, act.alpha, dh, got, 1e-6, strict=False, what="slerp bwd [2048,4096]")
    w = wl.wide(0).acts[0]
    dh = wl.normal_bf16(rng, (w.rows, w.cols))
    dres, dout, _ = run_slerp_bwd(w.x, w.r, w.alpha, dh, 1e-6, with_dalpha=False)
    rows = gu.sample_rows(w.rows, 48, 82)
    check_slerp_bwd(w.x[rows], w.r[rows], w.alpha, dh[rows], (dres[rows], dout[rows], None), 1e-6, strict=False,
                    what="slerp bwd [8192,7168]")


def test_slerp_backward_dalpha_deterministic_and_segmented():
    """dalpha is bitwise repeatable, and two segments sharing alpha give the
    column sums of their rows together."""
    rng = np.random.default_rng(83)
    C = 1024
    res, out, dh = (wl.normal_bf16(rng, (300, C)) for _ in range(3))
    alpha = wl.alpha_vec(rng, C)
    a1 = run_slerp_bwd(res, out, alpha, dh, 1e-6)[2]
    a2 = run_slerp_bwd(res, out, alpha, dh, 1e-6)[2]
    assert np.array_equal(a1, a2)
    al = gu.dev_f32(alpha)
    segs, outs = [], []
    for sl in (slice(0, 170), slice(170, 300)):
        d1 = torch.empty(sl.stop - sl.start, C, dtype=torch.float32, device="cuda")
        d2 = torch.empty_like(d1)
        segs.append(ds.AGSeg(x=gu.dev_bf16(res[sl]), r=gu.dev_bf16(out[sl]), dy=gu.dev_bf16(dh[sl]), dx=d1, dr=d2,
                             alpha=al))
        outs.append((d1, d2))
    da = torch.empty(C, dtype=torch.float32, device="cuda")
    ds.ds_slerp_rows_backward(segs, 1e-6, dalpha=da)
    torch.cuda.synchronize()
    got = (np.concatenate([gu.host_f32(d[0]) for d in outs]), np.concatenate([gu.host_f32(d[1]) for d in outs]),
           gu.host_f32(da))
    check_slerp_bwd(res, out, alpha, dh, got, 1e-6, strict=False, what="slerp bwd two segments")


def test_slerp_backward_special_alphas():
    """|alpha| = 0: out gets no gradient and dalpha is 0; |alpha| = 1: res gets none."""
    rng = np.random.default_rng(84)
    res, out, dh = (wl.normal_bf16(rng, (24, 512)) for _ in range(3))
    dres, dout, da = run_slerp_bwd(res, out, np.zeros(512, np.float32), dh, 1e-6)
    assert not dout.any() and not da.any()
    check_slerp_bwd(res, out, np.zeros(512, np.float32), dh, (dres, dout, da), 1e-6, strict=False)
    dres, dout, da = run_slerp_bwd(res, out, np.ones(512, np.float32), dh, 1e-6)
    assert not dres.any()
