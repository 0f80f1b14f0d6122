"""Pins for the oracle's backward of the activation rows (derived: the
TensorFold pages give tf_l2_rows and tf_slerp_rows forward only).

The backward is pinned against central finite differences of the forward
oracle's exact (pre-rounding) output, with the internal bf16 rounding points
switched off so that the forward is differentiable; against closed forms
(orthogonality of the l2 gradient to its row); against special cases of the
lerp weight (|alpha| = 0 or 1 leaves one input without gradient); and the
matrix drivers against the row functions.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from l2_row_b200 import workloads as wl


def _fd(f, x, h=1e-6):
    g = np.empty_like(x)
    for j in range(x.size):
        e = np.zeros_like(x)
        e[j] = h * max(1.0, abs(x[j]))
        g[j] = (f(x + e) - f(x - e)) / (2 * e[j])
    return g


@pytest.mark.parametrize("eps", [1e-6, 1e-3, 0.0])
@pytest.mark.parametrize("residual", [False, True])
def test_l2_backward_matches_central_differences(eps, residual):
    rng = np.random.default_rng(61)
    C = 24
    x = rng.standard_normal(C) * 0.3
    r = rng.standard_normal(C) * 0.3 if residual else None
    dy = rng.standard_normal(C)
    fl = oracle.OR_DROP_SUM_ROUND if residual else 0
    dx = oracle.l2_backward_row64(x, r, dy, eps=eps, flags=fl)
    fd = _fd(lambda v: oracle.l2_row64(v, r, eps=eps, flags=fl) @ dy, x)
    np.testing.assert_allclose(dx, fd, rtol=1e-6, atol=1e-8 * np.abs(dx).max())
    if residual:  # the residual gets the same gradient
        fdr = _fd(lambda v: oracle.l2_row64(x, v, eps=eps, flags=fl) @ dy, r)
        np.testing.assert_allclose(dx, fdr, rtol=1e-6, atol=1e-8 * np.abs(dx).max())


@pytest.mark.parametrize("eps", [1e-6, 1e-3])
def test_slerp_backward_matches_central_differences(eps):
    rng = np.random.default_rng(62)
    C = 20
    res = rng.standard_normal(C)
    out = rng.standard_normal(C)
    alpha = rng.uniform(-0.9, 0.9, C)
    alpha[alpha == 0] = 0.3
    dh = rng.standard_normal(C)
    fl = oracle.OR_DROP_SLERP_A | oracle.OR_DROP_SLERP_B
    dres, dout, da = oracle.slerp_backward_row64(res, out, alpha, dh, eps=eps, flags=fl)
    f = lambda a, b, al: oracle.slerp_row64(a, b, al, eps=eps, flags=fl) @ dh
    tol = dict(rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dres, _fd(lambda v: f(v, out, alpha), res), **tol)
    np.testing.assert_allclose(dout, _fd(lambda v: f(res, v, alpha), out), **tol)
    np.testing.assert_allclose(da, _fd(lambda v: f(res, out, v), alpha), **tol)


def test_l2_backward_uses_the_rounded_sum():
    """With a residual the forward normalises s = bf16(x + r); the backward
    differentiates through that rounded s (straight through the rounding)."""
    rng = np.random.default_rng(63)
    x = wl.normal_bf16(rng, (6, 40))
    r = wl.normal_bf16(rng, (6, 40))
    dy = wl.normal_bf16(rng, (6, 40))
    s = oracle.bf16_rne_array(wl.bf16_bits_to_f32(x).astype(np.float64) + wl.bf16_bits_to_f32(r))
    a = oracle.l2_rows_backward(x, r, dy)
    b = oracle.l2_rows_backward(s, None, dy)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("eps", [0.0, 1e-6, 1e-2])
def test_l2_backward_orthogonality_closed_form(eps):
    """s . dx = D - D S/(S+eps) over n = eps D / ((S + eps) n): zero at eps = 0."""
    rng = np.random.default_rng(64)
    x = wl.normal_bf16(rng, (10, 64))
    dy = wl.normal_bf16(rng, (10, 64))
    dx = oracle.l2_rows_backward(x, None, dy, eps=eps)
    s = wl.bf16_bits_to_f32(x).astype(np.float64)
    d = wl.bf16_bits_to_f32(dy).astype(np.float64)
    S, D = (s * s).sum(1), (s * d).sum(1)
    want = eps * D / ((S + eps) * np.sqrt(S + eps))
    got = (s * dx).sum(1)
    scale = np.linalg.norm(s, axis=1) * np.linalg.norm(dx, axis=1) + np.abs(want)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13 * scale.max())


def test_slerp_special_alphas():
    """|alpha| = 0: h depends on res only, so out gets no gradient (and
    neither does alpha, sign(0) = 0); |alpha| = 1: res gets none."""
    rng = np.random.default_rng(65)
    res = wl.normal_bf16(rng, (5, 48))
    out = wl.normal_bf16(rng, (5, 48))
    dh = wl.normal_bf16(rng, (5, 48))
    dres, dout, da = oracle.slerp_rows_backward(res, out, np.zeros(48, np.float32), dh)
    assert not dout.any() and not da.any() and dres.any()
    dres, dout, da = oracle.slerp_rows_backward(res, out, np.ones(48, np.float32), dh)
    assert not dres.any() and dout.any()
    # alpha of either sign: |alpha| is what the forward uses, the sign flips dalpha only
    al = rng.uniform(0.05, 0.5, 48).astype(np.float32)
    r1 = oracle.slerp_rows_backward(res, out, al, dh)
    r2 = oracle.slerp_rows_backward(res, out, -al, dh)
    assert np.array_equal(r1[0], r2[0]) and np.array_equal(r1[1], r2[1])
    assert np.array_equal(r1[2], -r2[2])


def test_matrix_drivers_match_row_functions():
    rng = np.random.default_rng(66)
    R, C = 7, 33
    x, r, dy = (wl.normal_bf16(rng, (R, C)) for _ in range(3))
    al = wl.alpha_vec(rng, C)
    f = lambda b: wl.bf16_bits_to_f32(b).astype(np.float64)
    dx = oracle.l2_rows_backward(x, r, dy, nthreads=3)
    dres, dout, da = oracle.slerp_rows_backward(x, r, al, dy, nthreads=4)
    acc = np.zeros(C)
    for i in range(R):
        np.testing.assert_array_equal(dx[i], oracle.l2_backward_row64(f(x[i]), f(r[i]), f(dy[i])))
        a, b, p = oracle.slerp_backward_row64(f(x[i]), f(r[i]), al.astype(np.float64), f(dy[i]))
        np.testing.assert_array_equal(dres[i], a)
        np.testing.assert_array_equal(dout[i], b)
        acc += p
    np.testing.assert_array_equal(da, acc)


def test_l2_backward_scale_invariance_eps0():
    """At eps = 0, x scaled by 2^k gives dx scaled by 2^-k exactly (y is
    scale-free, its gradient falls as 1/|x|)."""
    rng = np.random.default_rng(67)
    x = wl.normal_bf16(rng, (4, 32))
    dy = wl.normal_bf16(rng, (4, 32))
    dx = oracle.l2_rows_backward(x, None, dy, eps=0.0)
    for k in (-20, 7, 30):
        xk = wl.to_bf16_bits(np.ldexp(wl.bf16_bits_to_f32(x), k).astype(np.float32))
        dk = oracle.l2_rows_backward(xk, None, dy, eps=0.0)
        np.testing.assert_allclose(dk, np.ldexp(dx, -k), rtol=1e-15, atol=0)
