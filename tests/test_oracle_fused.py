"""Pins for the oracle's Dory activation rows (TensorFold PR #1260, the
norms.cu family: tf_gate_l2_rows and tf_swiglu_l2_rows).

They reduce to the l2 rows (pinned elsewhere by exact fixtures and closed
forms) where sigmoid and silu take exact or saturated values: sigmoid(0) is
exactly 1/2 (the pages' gate 4: "halves of integers, exact in fp32"), and a
large gate argument makes sigmoid 1 to far below a bf16 step.  The interval
forms must contain the point forms, keep fp32's exp range (0 reachable where
exp(-x) overflows fp32), and each control that drops one stated rounding
point must leave them.
"""
from __future__ import annotations

import numpy as np

import oracle
from l2_row_b200 import workloads as wl
from tests.checks import bf16_interval_violations


def _rows(seed, R=16, C=256):
    rng = np.random.default_rng(seed)
    return rng, wl.normal_bf16(rng, (R, C)), wl.normal_bf16(rng, (R, C))


def test_gate_at_zero_argument_is_l2_of_half_rows():
    """g = 0: sigmoid(0) = 1/2 exactly, the gated row is o/2 (exact in bf16),
    and at eps = 0 its l2 is that of o."""
    rng, o, _ = _rows(101)
    g = np.zeros_like(o)
    sg = rng.uniform(0.5, 2.0, o.shape[1]).astype(np.float32)
    assert np.array_equal(oracle.gate_l2_rows(o, g, sg, eps=0.0), oracle.l2_rows(o, None, eps=0.0))
    # integer rows (gate 4): the gated row is halves of integers
    x = wl.integer_rows(102, 8, 512)
    assert np.array_equal(oracle.gate_l2_rows(x, np.zeros_like(x), np.ones(512, np.float32), eps=0.0),
                          oracle.l2_rows(x, None, eps=0.0))


def test_gate_saturated_open_is_l2():
    """g sg >= 40: sigmoid = 1 - 4e-18, o times it rounds back to o."""
    rng, o, _ = _rows(103)
    g = wl.to_bf16_bits(np.full(o.shape, 48.0, np.float32))
    sg = np.ones(o.shape[1], np.float32)
    for eps in (1e-6, 0.0):
        assert np.array_equal(oracle.gate_l2_rows(o, g, sg, eps=eps), oracle.l2_rows(o, None, eps=eps))


def test_swiglu_saturated_gate_and_unit_up_is_l2_of_the_scaled_gate():
    """u suu = 1 and bf16(g sug) >= 24: silu(x) = x (1 - 4e-11) rounds back to
    x, so the row is l2(bf16(g sug))."""
    rng = np.random.default_rng(104)
    C = 256
    g = wl.to_bf16_bits(rng.uniform(24.0, 60.0, (8, C)).astype(np.float32))
    sug = rng.uniform(1.0, 1.5, C).astype(np.float32)
    u = wl.to_bf16_bits(np.ones((8, C), np.float32))
    suu = np.ones(C, np.float32)
    gs = oracle.bf16_rne_array(wl.bf16_bits_to_f32(g).astype(np.float64) * sug.astype(np.float64))
    for eps in (1e-6, 0.0):
        assert np.array_equal(oracle.swiglu_l2_rows(g, u, sug, suu, eps=eps), oracle.l2_rows(gs, None, eps=eps))


def test_swiglu_zero_gate_gives_zero_rows():
    rng, g, u = _rows(105)
    z = np.zeros_like(g)
    s = rng.uniform(0.5, 2.0, g.shape[1]).astype(np.float32)
    y = oracle.swiglu_l2_rows(z, u, s, s, eps=1e-6)
    assert not wl.bf16_bits_to_f32(y).any()


def test_intervals_contain_points():
    for seed in range(3):
        rng, a, b = _rows(106 + seed, 24, 512)
        s1 = rng.uniform(0.25, 4.0, 512).astype(np.float32)
        s2 = rng.uniform(0.25, 4.0, 512).astype(np.float32)
        y = oracle.gate_l2_rows(a, b, s1)
        assert not bf16_interval_violations(y, *oracle.gate_l2_rows_interval(a, b, s1)).any()
        y = oracle.swiglu_l2_rows(a, b, s1, s2)
        assert not bf16_interval_violations(y, *oracle.swiglu_l2_rows_interval(a, b, s1, s2)).any()


def test_gate_interval_keeps_fp32_exp_range():
    """g sg < -88.7: exp(-g sg) overflows fp32, so fp32 gates to exactly 0
    while float64 gives o e^(g sg) > 0; the interval must hold both."""
    C = 64
    o = wl.to_bf16_bits(np.ones((1, C), np.float32))
    g = wl.to_bf16_bits(np.full((1, C), -96.0, np.float32))
    g[0, :C // 2] = wl.to_bf16_bits(np.ones((1, C // 2), np.float32))[0]     # half the row gated normally
    sg = np.ones(C, np.float32)
    lo, hi = oracle.gate_l2_rows_interval(o, g, sg, eps=0.0)
    zero = np.zeros((1, C), np.uint16)
    point = oracle.gate_l2_rows(o, g, sg, eps=0.0)
    tail = slice(C // 2, C)
    assert not bf16_interval_violations(point[:, tail], lo[:, tail], hi[:, tail]).any()
    assert not bf16_interval_violations(zero[:, tail], lo[:, tail], hi[:, tail]).any()


def test_controls_leave_the_intervals():
    """Each control drops one rounding point the pages state; on the
    workload's rows every one of them lands outside the interval somewhere."""
    rng = np.random.default_rng(110)
    R, C = 64, 1024
    o, g = wl.normal_bf16(rng, (R, C)), wl.normal_bf16(rng, (R, C))
    sg = rng.uniform(0.5, 2.0, C).astype(np.float32)
    lo, hi = oracle.gate_l2_rows_interval(o, g, sg)
    y = oracle.gate_l2_rows(o, g, sg, flags=oracle.OR_DROP_GATED)
    assert bf16_interval_violations(y, lo, hi).any()
    u = wl.normal_bf16(rng, (R, C))
    sug = rng.uniform(0.5, 2.0, C).astype(np.float32)
    suu = rng.uniform(0.5, 2.0, C).astype(np.float32)
    lo, hi = oracle.swiglu_l2_rows_interval(g, u, sug, suu)
    for fl in (oracle.OR_DROP_SGATE, oracle.OR_DROP_SUP, oracle.OR_DROP_PRODUCT):
        y = oracle.swiglu_l2_rows(g, u, sug, suu, flags=fl)
        assert bf16_interval_violations(y, lo, hi).any(), hex(fl)


def test_threads_do_not_change_results():
    rng, a, b = _rows(111, 40, 300)
    s = rng.uniform(0.5, 2.0, 300).astype(np.float32)
    assert np.array_equal(oracle.gate_l2_rows(a, b, s, nthreads=1), oracle.gate_l2_rows(a, b, s, nthreads=6))
    assert np.array_equal(oracle.swiglu_l2_rows(a, b, s, s, nthreads=1),
                          oracle.swiglu_l2_rows(a, b, s, s, nthreads=5))


# ---------------------------------------------------- interior pins -----
#
# sigmoid and silu across the range the Dory rows use, against identities
# evaluated independently with Python's math module: sigmoid(z) =
# (1 + tanh(z/2)) / 2, sigmoid(z) + sigmoid(-z) = 1, silu(x) = x sigmoid(x).
# A wrong sign in exp, a dropped 1 or a swapped numerator fails them.

import math  # noqa: E402

Z = np.concatenate([np.linspace(-20.0, 20.0, 4001), np.random.default_rng(131).uniform(-20, 20, 2000),
                    [-1.2784645427610738, -1e-300, 0.0, 1e-300]])


def _sig_ref(z: float) -> float:
    """sigmoid by Python's math: (1 + tanh(z/2)) / 2 where it does not cancel
    (z >= 0), else e^z / (1 + e^z)."""
    if z >= 0:
        return 0.5 * (1.0 + math.tanh(0.5 * z))
    return math.exp(z) / (1.0 + math.exp(z))


def test_sigmoid_interior_matches_tanh_identity():
    for z in Z:
        s, ref = oracle.sigmoid(z), _sig_ref(z)
        assert abs(s - ref) <= 4.5e-16 * ref, (z, s, ref)
        assert abs(s + oracle.sigmoid(-z) - 1.0) <= 2.3e-16, z
    assert oracle.sigmoid(0.0) == 0.5


def test_silu_interior_is_x_times_sigmoid():
    for x in Z:
        ref = x * _sig_ref(x)
        assert abs(oracle.silu(x) - ref) <= 6e-16 * abs(ref) + 1e-300, (x, oracle.silu(x), ref)
    # silu's minimum near x0 = -1.27846...: silu'(x0) = 0, value -0.27846...
    x0 = -1.2784645427610738
    assert abs(oracle.silu(x0) - (-0.2784645427610738)) < 1e-15
    assert oracle.silu(x0 - 1e-4) > oracle.silu(x0) < oracle.silu(x0 + 1e-4)


def test_gate_and_swiglu_values_at_interior_points():
    """One element of each row: the unrounded values are o sigmoid(g sg) and
    silu(g sug) u suu, and the rounded ones their nearest bf16 (every
    rounding point applied)."""
    rng = np.random.default_rng(132)
    o = wl.bf16_bits_to_f32(wl.normal_bf16(rng, (500,))).astype(np.float64)
    g = wl.bf16_bits_to_f32(wl.normal_bf16(rng, (500,), 4.0)).astype(np.float64)
    s = rng.uniform(0.5, 2.0, 500).astype(np.float32).astype(np.float64)
    u = wl.bf16_bits_to_f32(wl.normal_bf16(rng, (500,))).astype(np.float64)
    s2 = rng.uniform(0.5, 2.0, 500).astype(np.float32).astype(np.float64)
    for i in range(500):
        v = o[i] * _sig_ref(g[i] * s[i])
        assert abs(oracle.gate_value(o[i], g[i], s[i], oracle.OR_DROP_GATED) - v) <= 1e-15 * abs(v) + 1e-300
        assert oracle.gate_value(o[i], g[i], s[i]) == oracle.bf16_value(oracle.bf16_rne(v)) or \
            abs(v * 256 / 2 ** math.floor(math.log2(abs(v))) % 1 - 0.5) < 1e-9
        flags = oracle.OR_DROP_SGATE | oracle.OR_DROP_SUP | oracle.OR_DROP_PRODUCT
        gs, us = g[i] * s[i], u[i] * s2[i]
        w = gs * _sig_ref(gs) * us
        assert abs(oracle.swiglu_value(g[i], u[i], s[i], s2[i], flags) - w) <= 2e-15 * abs(w) + 1e-300
        gs_b = oracle.bf16_value(oracle.bf16_rne(gs))
        us_b = oracle.bf16_value(oracle.bf16_rne(us))
        wr = gs_b * _sig_ref(gs_b) * us_b
        assert oracle.swiglu_value(g[i], u[i], s[i], s2[i]) == oracle.bf16_value(oracle.bf16_rne(wr)) or \
            abs(wr * 256 / 2 ** math.floor(math.log2(abs(wr))) % 1 - 0.5) < 1e-9
