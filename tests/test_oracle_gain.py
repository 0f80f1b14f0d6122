"""Pins for the oracle's row lengths, preserving gain and scalar gain
(DragonScale package description: options table, `gain` "scalar" and `init`
"preserve"; "Monitor" reads each layer's raw row lengths).

Row lengths are pinned by closed forms (rows of one repeated value); the
preserving gain by its purpose (the forward with it returns the raw rows);
the scalar gain's gradient by central finite differences of the forward in
g, and its per-row parts by the channel backward at equal gains.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from l2_row_b200 import workloads as wl


def test_row_lengths_closed_form():
    C = 256
    vals = np.array([1.0, -3.0, 0.5, 0.0], np.float32)
    w = np.repeat(vals[:, None], C, axis=1)
    n = oracle.row_norms(w, eps=0.0)
    np.testing.assert_array_equal(n, np.abs(vals).astype(np.float64) * 16.0)   # sqrt(256) = 16
    n = oracle.row_norms(w, eps=1e-6)
    np.testing.assert_allclose(n, np.sqrt(vals.astype(np.float64) ** 2 * C + 1e-6), rtol=1e-15)
    assert n[3] == np.sqrt(1e-6)


def test_preserving_gain_returns_the_raw_rows():
    rng = np.random.default_rng(71)
    w = wl.drifted_rows(rng, 12, 300, 0.02)
    for rho in (1.0, float(np.sqrt(300))):
        g = oracle.row_norms(w, eps=1e-6, div=rho)
        # the forward takes fp32 gains: W_eff equals w up to g's fp32 rounding
        weff = oracle.wn_forward(w, g.astype(np.float32), rho=rho, eps=1e-6)
        np.testing.assert_allclose(weff, w.astype(np.float64), rtol=2 ** -23, atol=0)


@pytest.mark.parametrize("bf16_gy", [False, True])
def test_scalar_gain_gradient_matches_finite_differences(bf16_gy):
    rng = np.random.default_rng(72)
    R, C = 9, 40
    w = wl.drifted_rows(rng, R, C, 1.0)
    gy = rng.standard_normal((R, C)).astype(np.float32)
    if bf16_gy:
        gy = wl.to_bf16_bits(gy)
    gyf = wl.bf16_bits_to_f32(gy) if bf16_gy else gy
    g, rho, eps = 1.75, 1.25, 1e-3
    _, parts, tot = oracle.wn_backward_scalar_gain(w, gy, g, rho=rho, eps=eps)

    # L(g) = sum GY . W_eff(g) is linear in g: a wide central step is exact
    # up to rounding (g +- h are exact in fp32)
    def L(gg):
        weff = oracle.wn_forward(w, np.full(R, gg, np.float32), rho=rho, eps=eps)
        return float((weff * gyf.astype(np.float64)).sum())

    h = 0.25
    fd = (L(g + h) - L(g - h)) / (2 * h)
    assert abs(tot - fd) <= 1e-12 * max(1.0, abs(fd))
    acc = 0.0
    for v in parts.tolist():      # the sum in row order
        acc += v
    assert tot == acc


def test_scalar_gain_parts_are_the_channel_gradient():
    rng = np.random.default_rng(73)
    w = wl.drifted_rows(rng, 7, 64, 0.1)
    gy = rng.standard_normal((7, 64)).astype(np.float32)
    gw_s, parts, _ = oracle.wn_backward_scalar_gain(w, gy, 0.75)
    gw_c, gg_c = oracle.wn_backward(w, gy, np.full(7, 0.75, np.float32))
    np.testing.assert_array_equal(gw_s, gw_c)
    np.testing.assert_array_equal(parts, gg_c)
