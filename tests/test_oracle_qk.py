"""Pins for the oracle's Dory q and k rows (TensorFold PR #1260,
tf_qk_rows_l2: rotate-half RoPE, then each head's L2 norm with eps on the
sum, then q times an fp32 scale vector).

The pins do not retype the oracle's formula.  At position 0 every rotation
is the identity, so the rows reduce to the l2 rows of each head (pinned by
exact fixtures elsewhere); the rotation itself is checked against complex
multiplication by exp(i theta) and against the relative-position property
of RoPE (q(p).k(p') depends on p - p' only) and the preservation of each
head's length; the interval forms must contain the point forms and the two
controls (the rotated head, q's normalized head) must leave them.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from l2_row_b200 import workloads as wl
from tests.checks import bf16_interval_violations

D = 64


def _heads(bits, head_dim):
    return bits.reshape(-1, head_dim)


def test_position_zero_is_the_l2_of_each_head():
    w = wl.qk_rows(1, rows=12, head_dim=D, hq=4, hk=2)
    pos = np.zeros(12, np.int32)
    qo, ko = oracle.qk_rows_l2(w.q, w.k, pos, w.inv, head_dim=D)
    assert np.array_equal(_heads(qo, D), oracle.l2_rows(_heads(w.q, D), None))
    assert np.array_equal(_heads(ko, D), oracle.l2_rows(_heads(w.k, D), None))
    # gate 4: integer heads, no rotation, exact fp32 sums
    x = wl.integer_rows(2, 8, 4 * 256)
    qo, ko = oracle.qk_rows_l2(x, x, np.zeros(8, np.int32), wl.rope_inv(256), head_dim=256, eps=0.0)
    ref = oracle.l2_rows(_heads(x, 256), None, eps=0.0)
    assert np.array_equal(_heads(qo, 256), ref) and np.array_equal(_heads(ko, 256), ref)


def test_power_of_two_scale_only_moves_the_exponent():
    w = wl.qk_rows(3, rows=6, head_dim=D, hq=2, hk=1)
    q0, _ = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, head_dim=D)
    q4, _ = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, np.full(2 * D, 4.0, np.float32), head_dim=D)
    f0, f4 = wl.bf16_bits_to_f32(q0), wl.bf16_bits_to_f32(q4)
    assert np.array_equal(f4, f0 * 4)


def _complex_rope(x_bits, pos, inv, head_dim, eps, scale=None):
    """The rotation as complex multiplication: z_i = x_i + i x_{i+h} times
    exp(i theta_i), theta = fp32(pos) * inv in fp32 (numpy's float32 product),
    then each head over sqrt(sum + eps), times scale."""
    h = head_dim // 2
    x = wl.bf16_bits_to_f32(x_bits).astype(np.float64)
    R = x.shape[0]
    x = x.reshape(R, -1, head_dim)
    th = (pos.astype(np.float32)[:, None] * inv[None, :]).astype(np.float64)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * th)[:, None, :]
    rot = np.concatenate([z.real, z.imag], axis=-1)
    y = rot / np.sqrt((rot * rot).sum(-1, keepdims=True) + eps)
    y = y.reshape(R, -1)
    return y if scale is None else y * scale.astype(np.float64)


@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_rotation_is_complex_multiplication(eps):
    """With the rounding points dropped, the exact outputs equal the complex
    form, at near and far (199,800+) positions alike: the angle is the fp32
    product, the halves pair i with i + D/2 and turn counter-clockwise."""
    w = wl.qk_rows(4, rows=30, head_dim=D, hq=3, hk=2)
    fl = oracle.OR_DROP_ROT | oracle.OR_DROP_QNORM
    _, _, qe, ke = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=D, eps=eps, flags=fl,
                                      exact=True)
    np.testing.assert_allclose(qe, _complex_rope(w.q, w.pos, w.inv, D, eps, w.q_scale), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(ke, _complex_rope(w.k, w.pos, w.inv, D, eps), rtol=1e-12, atol=1e-14)


def test_relative_position_and_length():
    """RoPE's defining property: with angles exact in fp32 (inv = 2^-j, small
    positions), q(p).k(p') is a function of p - p'; each rotated head keeps
    its length (unit after the norm at eps = 0)."""
    h = D // 2
    inv = np.ldexp(np.ones(h, np.float32), -np.arange(h)).astype(np.float32)
    rng = np.random.default_rng(5)
    qh = wl.normal_bf16(rng, (1, D))
    kh = wl.normal_bf16(rng, (1, D))
    fl = oracle.OR_DROP_ROT | oracle.OR_DROP_QNORM

    def rot(bits, p):
        _, _, e, _ = oracle.qk_rows_l2(bits, kh, np.array([p], np.int32), inv, head_dim=D, eps=0.0, flags=fl,
                                       exact=True)
        return e[0]

    for p, pp, d in ((3, 10, 5), (0, 7, 100), (40, 1, 17)):
        a = rot(qh, p) @ rot(kh, pp)
        b = rot(qh, p + d) @ rot(kh, pp + d)
        assert abs(a - b) < 1e-13, (p, pp, d, a, b)
        assert abs(rot(qh, p) @ rot(qh, p) - 1.0) < 1e-14


def test_intervals_contain_points():
    for seed, D_, hq, hk in ((6, 64, 4, 2), (7, 256, 16, 4), (8, 128, 2, 2)):
        w = wl.qk_rows(seed, rows=24, head_dim=D_, hq=hq, hk=hk)
        for sc in (None, w.q_scale):
            qo, ko = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, sc, head_dim=D_)
            ql, qh, kl, kh = oracle.qk_rows_l2_interval(w.q, w.k, w.pos, w.inv, sc, head_dim=D_)
            assert not bf16_interval_violations(qo, ql, qh).any()
            assert not bf16_interval_violations(ko, kl, kh).any()


def test_controls_leave_the_intervals():
    """The pages' workload (head dim 256, 16 query heads over 4, a third of
    the rows past 199,800): dropping the rotated head's rounding or q's
    normalized head's rounding lands outside the interval somewhere."""
    w = wl.qk_rows(9, rows=48)
    ql, qh, kl, kh = oracle.qk_rows_l2_interval(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=256, nthreads=4)
    qo, ko = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=256, flags=oracle.OR_DROP_ROT,
                               nthreads=4)
    assert bf16_interval_violations(qo, ql, qh).any() and bf16_interval_violations(ko, kl, kh).any()
    qo, _ = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=256, flags=oracle.OR_DROP_QNORM,
                              nthreads=4)
    assert bf16_interval_violations(qo, ql, qh).any()


def test_far_positions_need_the_fp32_angle():
    """At 199,800 the fp32 angle differs from the exact product by up to
    ~0.008 rad: the far rows' outputs differ from those of a float64 angle,
    the near rows' hardly."""
    w = wl.qk_rows(10, rows=12, head_dim=D, hq=2, hk=1)
    fl = oracle.OR_DROP_ROT | oracle.OR_DROP_QNORM
    _, _, qe, _ = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, head_dim=D, flags=fl, exact=True)
    h = D // 2
    x = wl.bf16_bits_to_f32(w.q).astype(np.float64).reshape(12, -1, D)
    th = w.pos.astype(np.float64)[:, None] * w.inv.astype(np.float64)[None, :]
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * th)[:, None, :]
    rot = np.concatenate([z.real, z.imag], axis=-1)
    y64 = (rot / np.sqrt((rot * rot).sum(-1, keepdims=True) + 1e-6)).reshape(12, -1)
    far = w.pos >= 199_800
    assert np.abs(qe[far] - y64[far]).max() > 1e-4
    assert np.abs(qe[~far] - y64[~far]).max() < 1e-6


def test_threads_do_not_change_results():
    w = wl.qk_rows(11, rows=40, head_dim=D, hq=4, hk=2)
    a = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=D, nthreads=1)
    b = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=D, nthreads=7)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))


def test_intervals_contain_points_at_extremes():
    """Heads of huge, tiny and mixed magnitudes, zero heads, and positions
    up to 2^24 (angles far past 2 pi): the interval still holds the point."""
    rng = np.random.default_rng(12)
    D, R = 64, 6
    inv = wl.rope_inv(D)
    pos = np.array([0, 1, 199_800, 1 << 20, (1 << 24) - 1, 12345], np.int32)
    for scale in (1e30, 1e-30, 1.0):
        x = (rng.standard_normal((R, 2 * D)) * scale).astype(np.float32)
        x[1, :D] = 0.0                                   # one zero head
        q = wl.to_bf16_bits(x)
        k = wl.to_bf16_bits((rng.standard_normal((R, D)) * scale).astype(np.float32))
        for eps in (1e-6, 0.0):
            qo, ko = oracle.qk_rows_l2(q, k, pos, inv, head_dim=D, eps=eps)
            ql, qh, kl, kh = oracle.qk_rows_l2_interval(q, k, pos, inv, head_dim=D, eps=eps)
            fin = ~np.isnan(wl.bf16_bits_to_f32(qo))
            assert not bf16_interval_violations(qo[fin], ql[fin], qh[fin]).any(), (scale, eps)
            fin = ~np.isnan(wl.bf16_bits_to_f32(ko))
            assert not bf16_interval_violations(ko[fin], kl[fin], kh[fin]).any(), (scale, eps)
