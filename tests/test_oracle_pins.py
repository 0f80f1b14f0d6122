"""Pins for the float64 oracle: exact fixtures, closed forms, invariants,
central finite differences and negative controls.

Sources: DragonScale package description ("What DragonScale changes", eq.
W_eff and eq. dL/dW; "Why scales drift", the free scale direction;
"Optimizer", rescale after the step) and TensorFold PR #1260 (tf_l2_rows,
tf_slerp_rows and their rounding points and controls).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from l2_row_b200 import workloads as wl
from tests.checks import SPREAD, bf16_interval_violations, bf16_key, bf16_ulp_violations
from tests.golden_io import act_cases, wn_cases


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.max(np.abs(a - b) / np.maximum(np.abs(b), 1e-300)) if a.size else 0.0


# ---------------------------------------------------------------- fixtures --

@pytest.mark.parametrize("case", wn_cases(), ids=lambda c: ",".join(str(v) for v in c["w"]))
def test_golden_weight_rows(case):
    w = np.array([[float(v) for v in case["w"]]], np.float32)
    g = np.array([float(case["g"])], np.float32)
    gy = np.array([[float(v) for v in case["gy"]]], np.float32)
    rho, eps = float(case["rho"]), float(case["eps"])
    weff = oracle.wn_forward(w, g, rho=rho, eps=eps)[0]
    gw, gg = oracle.wn_backward(w, gy, g, rho=rho, eps=eps)
    rn = oracle.row_renorm(w, rho=rho, eps=eps)[0]
    np.testing.assert_allclose(weff, [float(v) for v in case["weff"]], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(gw[0], [float(v) for v in case["grad_w"]], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(gg[0], float(case["grad_g"]), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(rn, [float(v) for v in case["renorm"]], rtol=1e-15, atol=1e-15)


def test_golden_printed_form_differs_with_eps():
    """The eps = 11 fixture separates the exact derivative from the printed eps-free projection."""
    w = np.array([[3, 4]], np.float32)
    gy = np.array([[1, 0]], np.float32)
    gw, _ = oracle.wn_backward(w, gy, None, eps=11.0, flags=oracle.OR_BWD_PRINTED)
    np.testing.assert_allclose(gw[0], [8 / 75, -2 / 25], rtol=1e-14)


@pytest.mark.parametrize("case", act_cases(), ids=lambda c: c["op"] + ":" + ",".join(str(v) for v in c["x"]))
def test_golden_activation_rows(case):
    x = wl.to_bf16_bits(np.array([[float(v) for v in case["x"]]], np.float32))
    assert np.array_equal(wl.bf16_bits_to_f32(x)[0], [float(v) for v in case["x"]])  # exact inputs
    eps = float(case["eps"])
    if case["op"] == "l2":
        r = None if case["r"] is None else wl.to_bf16_bits(np.array([[float(v) for v in case["r"]]], np.float32))
        y = oracle.l2_rows(x, r, eps=eps)[0]
    else:
        out = wl.to_bf16_bits(np.array([[float(v) for v in case["r"]]], np.float32))
        alpha = np.array([float(v) for v in case["alpha"]], np.float32)
        y = oracle.slerp_rows(x, out, alpha, eps=eps)[0]
    assert [int(v) for v in y] == case["bits"]


def test_golden_residual_rounding_point_is_visible():
    x = wl.to_bf16_bits(np.array([[1, 1]], np.float32))
    r = wl.to_bf16_bits(np.array([[0.01953125, 0]], np.float32))
    y = oracle.l2_rows(x, r, eps=0.0, flags=oracle.OR_DROP_SUM_ROUND)[0]
    assert [int(v) for v in y] == [0x3F37, 0x3F33]


# ------------------------------------------------------------ closed forms --

@pytest.fixture(scope="module")
def tiny():
    return wl.tiny(0)


def test_forward_row_norm_closed_form(tiny):
    """||W_eff_r|| = |g_r| rho sqrt(S) / sqrt(S + eps)."""
    s = tiny.weights[0]
    for rho in (1.0, float(np.sqrt(128))):
        out = oracle.wn_forward(s.w, s.g, rho=rho, eps=tiny.eps)
        w64 = s.w.astype(np.float64)
        S = np.einsum("ij,ij->i", w64, w64)
        want = np.abs(s.g.astype(np.float64)) * rho * np.sqrt(S) / np.sqrt(S + tiny.eps)
        assert _rel(np.linalg.norm(out, axis=1), want) < 1e-14


def test_forward_scale_invariance_eps0():
    """The free scale direction: W_eff(c w) = W_eff(w) for any c > 0 (eps = 0)."""
    rng = np.random.default_rng(3)
    w = rng.standard_normal(257)
    base = oracle.wn_forward_row64(w, 1.7, eps=0.0)
    for c in (1e-3, 0.7, 3.0, 1e4):
        assert _rel(oracle.wn_forward_row64(c * w, 1.7, eps=0.0), base) < 1e-14


def test_forward_scale_with_eps_closed_form():
    rng = np.random.default_rng(4)
    w = rng.standard_normal(64) * 1e-3
    eps = 1e-6
    S = float(w @ w)
    base = oracle.wn_forward_row64(w, 1.0, eps=eps)
    for c in (0.1, 2.0, 50.0):
        factor = c * np.sqrt(S + eps) / np.sqrt(c * c * S + eps)
        assert _rel(oracle.wn_forward_row64(c * w, 1.0, eps=eps), base * factor) < 1e-14


def test_backward_orthogonality_closed_form(tiny):
    """w . grad_w = g rho eps D / n^3; exactly 0 at eps = 0 (gradient tangent to the row)."""
    s = tiny.weights[0]
    gw, _ = oracle.wn_backward(s.w, s.gy, s.g, eps=tiny.eps)
    w64, gy64 = s.w.astype(np.float64), s.gy.astype(np.float64)
    S = np.einsum("ij,ij->i", w64, w64)
    D = np.einsum("ij,ij->i", w64, gy64)
    n = np.sqrt(S + tiny.eps)
    want = s.g * tiny.eps * D / n ** 3
    dot = np.einsum("ij,ij->i", w64, gw)
    scale = np.linalg.norm(w64, axis=1) * np.linalg.norm(gw, axis=1)
    assert np.all(np.abs(dot - want) <= 1e-12 * scale)
    gw0, _ = oracle.wn_backward(s.w, s.gy, s.g, eps=0.0)
    dot0 = np.einsum("ij,ij->i", w64, gw0)
    assert np.all(np.abs(dot0) <= 1e-13 * np.linalg.norm(w64, axis=1) * np.linalg.norm(gw0, axis=1))


def test_norm_growth_law_for_free_scale():
    """For a scale-free w (<grad, w> = 0) one step w' = w - lr*grad gives
    ||w'||^2 = ||w||^2 + lr^2 ||grad||^2: the drift the method removes."""
    rng = np.random.default_rng(5)
    w = rng.standard_normal(128)
    gy = rng.standard_normal(128)
    gw, _ = oracle.wn_backward_row64(w, gy, 1.3, eps=0.0)
    lr = 0.05
    w2 = w - lr * gw
    assert abs(w2 @ w2 - (w @ w + lr * lr * (gw @ gw))) < 1e-12 * (w @ w)


# ---------------------------------------------------- finite differences --

def _fd_check(R, C, seed, eps, rho=1.0, flags=0):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((R, C)) * np.exp(rng.standard_normal((R, 1)))
    gy = rng.standard_normal((R, C))
    g = rng.uniform(0.5, 2.0, R)
    worst_w = worst_g = 0.0
    for r in range(R):
        gw, gg = oracle.wn_backward_row64(w[r], gy[r], g[r], rho=rho, eps=eps, flags=flags)
        L = lambda wr, gr: float(gy[r] @ oracle.wn_forward_row64(wr, gr, rho=rho, eps=eps))
        fd = np.empty(C)
        for j in range(C):
            h = 1e-6 * max(1.0, abs(w[r, j]))
            wp, wm = w[r].copy(), w[r].copy()
            wp[j] += h
            wm[j] -= h
            fd[j] = (L(wp, g[r]) - L(wm, g[r])) / (2 * h)
        hg = 1e-6 * max(1.0, abs(g[r]))
        fdg = (L(w[r], g[r] + hg) - L(w[r], g[r] - hg)) / (2 * hg)
        scale = np.max(np.abs(fd))
        worst_w = max(worst_w, np.max(np.abs(gw - fd)) / scale)
        worst_g = max(worst_g, abs(gg - fdg) / max(abs(fdg), 1e-300))
    return worst_w, worst_g


@pytest.mark.parametrize("R,C,eps,rho", [(8, 16, 1e-6, 1.0), (8, 16, 0.5, 2.0), (4, 128, 1e-6, 1.0)])
def test_backward_matches_central_differences(R, C, eps, rho):
    ww, wg = _fd_check(R, C, 11, eps, rho)
    assert ww < 1e-7 and wg < 1e-7, (ww, wg)


def test_backward_config1_central_differences(tiny):
    """All 64 x 128 entries of the tiny weight, at its eps."""
    s = tiny.weights[0]
    w = s.w.astype(np.float64)
    worst = 0.0
    for r in range(0, 64, 4):  # every 4th row keeps the CPU suite fast; all 128 columns each
        gw, gg = oracle.wn_backward_row64(w[r], s.gy[r].astype(np.float64), float(s.g[r]), eps=tiny.eps)
        L = lambda wr: float(s.gy[r].astype(np.float64) @ oracle.wn_forward_row64(wr, float(s.g[r]), eps=tiny.eps))
        fd = np.empty(128)
        for j in range(128):
            h = 1e-6 * max(1.0, abs(w[r, j]))
            wp, wm = w[r].copy(), w[r].copy()
            wp[j] += h
            wm[j] -= h
            fd[j] = (L(wp) - L(wm)) / (2 * h)
        worst = max(worst, np.max(np.abs(gw - fd)) / np.max(np.abs(fd)))
    assert worst < 1e-7


def test_printed_eps_free_form_fails_fd_on_small_rows():
    """Control for the eps reading: the eps-free projection misses the FD
    gradient on rows whose squared norm is near eps."""
    rng = np.random.default_rng(12)
    w = rng.standard_normal(16) * 3e-4   # S ~ 1.4e-6, comparable to eps = 1e-6
    gy = rng.standard_normal(16)
    eps = 1e-6
    gw_ok, _ = oracle.wn_backward_row64(w, gy, 1.0, eps=eps)
    gw_bad, _ = oracle.wn_backward_row64(w, gy, 1.0, eps=eps, flags=oracle.OR_BWD_PRINTED)
    L = lambda wr: float(gy @ oracle.wn_forward_row64(wr, 1.0, eps=eps))
    fd = np.array([(L(w + h * e) - L(w - h * e)) / (2 * h)
                   for e, h in ((np.eye(16)[j], 1e-10) for j in range(16))])
    s = np.max(np.abs(fd))
    assert np.max(np.abs(gw_ok - fd)) / s < 1e-5
    assert np.max(np.abs(gw_bad - fd)) / s > 1e-2


# -------------------------------------------------------------- renorm --

def test_renorm_idempotent_and_forward_preserving(tiny):
    s = tiny.weights[0]
    once = oracle.row_renorm(s.w, eps=0.0)
    twice = oracle.row_renorm(once.astype(np.float32), eps=0.0)
    # renorm of the fp32-rounded unit rows changes them by at most their own rounding
    assert _rel(twice, once) < 2e-7
    f0 = oracle.wn_forward(s.w, s.g, eps=0.0)
    f1 = oracle.wn_forward(once.astype(np.float32), s.g, eps=0.0)
    assert _rel(f1, f0) < 2e-7
    # in f64 (no fp32 round trip) the identity is exact up to f64 rounding
    r64 = np.array([oracle.wn_forward_row64(oracle.wn_forward_row64(s.w[i].astype(np.float64), 1.0, eps=0.0),
                                            1.0, eps=0.0) for i in range(4)])
    assert _rel(r64, once[:4]) < 1e-15


def test_renorm_radius_embedding():
    rng = np.random.default_rng(8)
    w = rng.standard_normal((3, 768)).astype(np.float32)
    out = oracle.row_renorm(w, rho=np.sqrt(768.0), eps=0.0)
    assert _rel(np.sqrt(np.mean(out ** 2, axis=1)), np.ones(3)) < 1e-14   # unit RMS rows


def test_zero_rows():
    z = np.zeros((2, 8), np.float32)
    assert np.all(oracle.wn_forward(z, None, eps=1e-6) == 0)
    assert np.all(np.isnan(oracle.wn_forward(z, None, eps=0.0)))
    y = oracle.l2_rows(np.zeros((2, 8), np.uint16), eps=1e-6)
    assert np.all(y == 0)
    y0 = oracle.l2_rows(np.zeros((2, 8), np.uint16), eps=0.0)
    assert np.all((y0 & 0x7F80) == 0x7F80) and np.all(y0 & 0x7F)


def test_nonfinite_propagation():
    x = wl.to_bf16_bits(np.array([[1.0, np.inf, 2.0, 0.0], [1.0, np.nan, 2.0, 0.0]], np.float32))
    y = oracle.l2_rows(x, eps=1e-6)
    # inf row: S = inf, finite entries -> 0, the inf entry -> inf/inf = NaN
    assert y[0, 0] == 0 and y[0, 2] == 0 and y[0, 3] == 0 and (y[0, 1] & 0x7FFF) > 0x7F80
    assert np.all((y[1] & 0x7FFF) > 0x7F80)


# --------------------------------------------------------- activation rows --

@pytest.fixture(scope="module")
def act():
    return wl.tiny(0).acts[0]


def test_l2_zero_residual_equals_none(act):
    y0 = oracle.l2_rows(act.x, None, eps=1e-6)
    y1 = oracle.l2_rows(act.x, np.zeros_like(act.r), eps=1e-6)
    assert np.array_equal(y0, y1)


def test_l2_exact_output_norm(act):
    _, ye = oracle.l2_rows(act.x, act.r, eps=1e-6, exact=True)
    s = wl.bf16_bits_to_f32(wl.to_bf16_bits(wl.bf16_bits_to_f32(act.x) + wl.bf16_bits_to_f32(act.r)))
    S = np.einsum("ij,ij->i", s.astype(np.float64), s.astype(np.float64))
    assert _rel(np.linalg.norm(ye, axis=1), np.sqrt(S / (S + 1e-6))) < 1e-14


def test_slerp_special_alphas(act):
    a = oracle.l2_rows(act.x, eps=1e-6)
    b = oracle.l2_rows(act.r, eps=1e-6)
    C = act.cols
    h0 = oracle.slerp_rows(act.x, act.r, np.zeros(C, np.float32), eps=1e-6)
    assert np.array_equal(h0, oracle.l2_rows(a, eps=1e-6))
    signs = np.where(np.arange(C) % 2 == 0, 1.0, -1.0).astype(np.float32)
    h1 = oracle.slerp_rows(act.x, act.r, signs, eps=1e-6)
    assert np.array_equal(h1, oracle.l2_rows(b, eps=1e-6))
    hs = oracle.slerp_rows(act.x, act.x, act.alpha, eps=1e-6)
    assert np.array_equal(hs, oracle.l2_rows(a, eps=1e-6))
    # only |alpha| enters
    assert np.array_equal(oracle.slerp_rows(act.x, act.r, act.alpha, eps=1e-6),
                          oracle.slerp_rows(act.x, act.r, -act.alpha, eps=1e-6))


def test_threads_do_not_change_results(act):
    w = wl.mlp_pair(0).weights[0]
    a = oracle.wn_backward(w.w[:64], w.gy[:64], w.g[:64], nthreads=1)
    b = oracle.wn_backward(w.w[:64], w.gy[:64], w.g[:64], nthreads=5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.array_equal(oracle.slerp_rows(act.x, act.r, act.alpha, nthreads=1),
                          oracle.slerp_rows(act.x, act.r, act.alpha, nthreads=3))


def test_integer_rows_exceed_fp16_but_not_fp32():
    """The exact-sum control set: sums of squares above fp16's 65504 and below 2^24."""
    x = wl.integer_rows(3, 16, 4096)
    v = wl.bf16_bits_to_f32(x).astype(np.int64)
    S = np.sum(v * v, axis=1)
    assert np.all(S > 65504) and np.all(S < 2 ** 24)


# -------------------------------------------------------- negative controls --

def test_interval_forms_bracket_point_forms():
    act = wl.activations(1, rows=64, cols=1024).acts[0]
    y = oracle.l2_rows(act.x, act.r)
    lo0, hi0 = oracle.l2_rows_interval(act.x, act.r, delta=0.0)
    assert np.array_equal(lo0, y) and np.array_equal(hi0, y)
    lo, hi = oracle.l2_rows_interval(act.x, act.r, delta=SPREAD)
    assert not bf16_interval_violations(y, lo, hi).any()
    assert np.mean(lo == hi) > 0.99          # sharp: almost every output is pinned to one value
    h = oracle.slerp_rows(act.x, act.r, act.alpha)
    lo0, hi0 = oracle.slerp_rows_interval(act.x, act.r, act.alpha, delta=0.0)
    assert np.array_equal(lo0, h) and np.array_equal(hi0, h)
    lo, hi = oracle.slerp_rows_interval(act.x, act.r, act.alpha, delta=SPREAD)
    assert not bf16_interval_violations(h, lo, hi).any()
    assert np.mean(lo == hi) > 0.95
    # wider ranges only where slerp's a or b sits on a halfway point and the
    # lerp cancels (t near 0): there either rounding of a is a legitimate fp32 outcome
    assert np.mean(bf16_key(hi) - bf16_key(lo) <= 1) > 0.999


def test_controls_escape_the_sharp_interval():
    """Each control drops one rounding point or moves eps.  Within 1 ulp it can
    hide (dropping a rounding point moves a result by at most ~half an ulp), so
    the controls are decided by the interval check: on the control inputs each
    must put at least one row outside the definition's interval."""
    act = wl.activations(0, rows=256, cols=4096).acts[0]
    lo, hi = oracle.l2_rows_interval(act.x, act.r, delta=SPREAD)
    drop = oracle.l2_rows(act.x, act.r, flags=oracle.OR_DROP_SUM_ROUND)
    assert bf16_interval_violations(drop, lo, hi).any(axis=1).any()
    lo, hi = oracle.slerp_rows_interval(act.x, act.r, act.alpha, delta=SPREAD)
    for f in (oracle.OR_DROP_SLERP_A, oracle.OR_DROP_SLERP_B):
        ctl = oracle.slerp_rows(act.x, act.r, act.alpha, flags=f)
        assert bf16_interval_violations(ctl, lo, hi).any(axis=1).any(), f
    small = wl.small_norm_rows(5, 64, 4096)
    b = oracle.l2_rows(small)
    lo, hi = oracle.l2_rows_interval(small, delta=SPREAD)
    for f in (oracle.OR_EPS_OUTSIDE, oracle.OR_EPS_ZERO):
        ctl = oracle.l2_rows(small, flags=f)
        assert bf16_ulp_violations(ctl, b).any(axis=1).any(), f    # eps moves are large: 1 ulp catches them
        assert bf16_interval_violations(ctl, lo, hi).any(axis=1).any(), f


def test_eps_sensitivity_in_f64():
    """A 1e-10 relative change of eps is visible in the f64 forward on rows
    whose squared norm is near eps."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((4, 64)) * 1.25e-4).astype(np.float32)
    a = oracle.wn_forward(w, None, eps=1e-6)
    b = oracle.wn_forward(w, None, eps=1e-6 * (1 + 1e-10))
    assert _rel(b, a) > 1e-12
