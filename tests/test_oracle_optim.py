"""Pins for the oracle's optimizer companions of method "rescale"
(DragonScale package description, "Optimizer"): the gradient projection
before the step and the momentum projection fused with the renorm after it.

Each pin comes from outside the function it checks: exact rationals derived
by hand (tests/golden/optim_exact.txt), numpy's least-squares solver for the
component along the row, the backward (itself pinned by central finite
differences, which equals the projection scaled by g rho / n), closed forms
and invariants.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from l2_row_b200 import workloads as wl
from tests.golden_io import optim_cases


def _rows(seed, R, C, scale=1.0):
    rng = np.random.default_rng(seed)
    w = wl.drifted_rows(rng, R, C, scale)
    G = rng.standard_normal((R, C), dtype=np.float32)
    return w, G


@pytest.mark.parametrize("case", optim_cases(), ids=lambda c: ",".join(str(v) for v in c["w"]) + f"|eps={c['eps']}")
def test_golden_optimizer_rows(case):
    w = np.array([[float(v) for v in case["w"]]], np.float32)
    G = np.array([[float(v) for v in case["G"]]], np.float32)
    eps, rho = float(case["eps"]), float(case["rho"])
    P = oracle.grad_project(w, G, eps=eps)[0]
    np.testing.assert_allclose(P, [float(v) for v in case["P"]], rtol=1e-15, atol=1e-15)
    wo, mo = oracle.renorm_momentum(w, G, rho=rho, eps=eps)
    np.testing.assert_allclose(mo[0], [float(v) for v in case["P"]], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(wo[0], [float(v) for v in case["renorm"]], rtol=1e-15, atol=1e-15)


def test_projection_is_least_squares_residual():
    """At eps = 0 the result is G minus its least-squares fit by the row
    (numpy's solver), i.e. the orthogonal projection onto the row's complement."""
    w, G = _rows(31, 16, 48)
    P = oracle.grad_project(w, G, eps=0.0)
    for r in range(w.shape[0]):
        A = w[r].astype(np.float64)[:, None]
        c, *_ = np.linalg.lstsq(A, G[r].astype(np.float64), rcond=None)
        ref = G[r] - c[0] * w[r].astype(np.float64)
        np.testing.assert_allclose(P[r], ref, rtol=0, atol=1e-12 * np.linalg.norm(G[r]))


@pytest.mark.parametrize("eps", [0.0, 1e-6, 1e-2])
def test_projection_equals_backward_times_norm(eps):
    """The backward with g = rho = 1 is (1/n)(GY - w D/(S+eps)): the same
    projection divided by n = sqrt(S + eps) (the backward is pinned by
    central finite differences)."""
    w, G = _rows(32, 12, 40, scale=0.05)
    P = oracle.grad_project(w, G, eps=eps)
    gw, _ = oracle.wn_backward(w, G, None, eps=eps)
    n = np.sqrt((w.astype(np.float64) ** 2).sum(1, keepdims=True) + eps)
    np.testing.assert_allclose(P, gw * n, rtol=1e-13, atol=1e-13 * np.abs(P).max())


@pytest.mark.parametrize("eps", [0.0, 1e-6, 1e-3])
def test_projection_orthogonality_closed_form(eps):
    """w . P(G) = D - D S/(S+eps) = eps D/(S+eps): zero at eps = 0."""
    w, G = _rows(33, 20, 64, scale=0.05)
    P = oracle.grad_project(w, G, eps=eps)
    w64, G64 = w.astype(np.float64), G.astype(np.float64)
    S = (w64 ** 2).sum(1)
    D = (w64 * G64).sum(1)
    lhs = (w64 * P).sum(1)
    scale = np.linalg.norm(w64, axis=1) * np.linalg.norm(G64, axis=1)
    np.testing.assert_allclose(lhs, eps * D / (S + eps), rtol=0, atol=1e-13 * scale.max())


def test_projection_idempotent_at_eps0():
    w, G = _rows(34, 10, 33)
    P = oracle.grad_project(w, G, eps=0.0)
    PP = oracle.grad_project(w, P.astype(np.float32), eps=0.0)
    # P enters rounded to fp32; projecting again removes only that rounding's component
    Pf = P.astype(np.float32).astype(np.float64)
    np.testing.assert_allclose(PP, Pf, rtol=0, atol=1e-6 * np.abs(Pf).max())


def test_projection_scale_invariant_in_w_at_eps0():
    """Only the row's direction matters: P(c w, G) = P(w, G) for c > 0 (eps = 0)."""
    w, G = _rows(35, 8, 24)
    P = oracle.grad_project(w, G, eps=0.0)
    for c in (2.0 ** -20, 0.3, 7.0, 2.0 ** 30):
        Pc = oracle.grad_project((w.astype(np.float64) * c).astype(np.float32), G, eps=0.0)
        np.testing.assert_allclose(Pc, P, rtol=0, atol=1e-6 * np.abs(P).max())


def test_momentum_pieces_match_renorm_and_projection():
    """The fused call is the renorm of w and the projection of m, both
    from the row as the step left it."""
    w, m = _rows(36, 14, 50)
    for rho, eps in ((1.0, 1e-6), (np.sqrt(50.0), 0.0), (2.0, 1e-2)):
        wo, mo = oracle.renorm_momentum(w, m, rho=rho, eps=eps)
        np.testing.assert_allclose(wo, oracle.row_renorm(w, rho=rho, eps=eps), rtol=0, atol=0)
        np.testing.assert_allclose(mo, oracle.grad_project(w, m, eps=eps), rtol=0, atol=0)
        # the renormed row has length rho sqrt(S/(S+eps))
        S = (w.astype(np.float64) ** 2).sum(1)
        np.testing.assert_allclose(np.linalg.norm(wo, axis=1), rho * np.sqrt(S / (S + eps)), rtol=1e-14)


def test_eps_zero_control_flag():
    w, G = _rows(37, 4, 16, scale=1e-3)
    np.testing.assert_allclose(oracle.grad_project(w, G, eps=1e-6, flags=oracle.OR_EPS_ZERO),
                               oracle.grad_project(w, G, eps=0.0), rtol=0, atol=0)
    # small rows: eps visibly changes the result
    d = np.abs(oracle.grad_project(w, G, eps=1e-6) - oracle.grad_project(w, G, eps=0.0)).max()
    assert d > 1e-3 * np.abs(G).max()


def test_threads_do_not_change_results():
    w, G = _rows(38, 64, 40)
    a = oracle.grad_project(w, G, nthreads=1)
    b = oracle.grad_project(w, G, nthreads=7)
    assert np.array_equal(a, b)
    wa, ma = oracle.renorm_momentum(w, G, nthreads=1)
    wb, mb = oracle.renorm_momentum(w, G, nthreads=5)
    assert np.array_equal(wa, wb) and np.array_equal(ma, mb)
