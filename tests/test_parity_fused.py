"""GPU parity of Dory's gated and SwiGLU l2 rows (TensorFold PR #1260,
tf_gate_l2_rows and tf_swiglu_l2_rows) against the float64 oracle.

The kernels evaluate sigmoid and silu in fp32 with CUDA's expf, so every
output must lie in the oracle's interval (the fp32 spread of each step, exp's
ulps, fp32's exp range) and within 1 bf16 ulp of the oracle's point value
unless the interval allows more -- the same rule as the slerp rows.  Inputs:
o, g, u ~ N(0,1) bf16 and scale vectors ~ U(0.5, 2) fp32 (the pages form them
on the host and give no values).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests import gpu_util as gu
from tests.checks import bf16_interval_violations

pytestmark = pytest.mark.gpu

PATHS = [ds.DS_PATH_AUTO, ds.DS_PATH_WARP, ds.DS_PATH_CTA]
PATH_IDS = ["auto", "warp", "cta"]


def _inputs(rng, R, C):
    a, b = wl.normal_bf16(rng, (R, C)), wl.normal_bf16(rng, (R, C))
    sa = rng.uniform(0.5, 2.0, C).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, C).astype(np.float32)
    return a, b, sa, sb


def run(swiglu, a, b, sa, sb, eps):
    R, C = a.shape
    ad, bd = gu.dev_bf16(a), gu.dev_bf16(b)
    y = torch.empty_like(ad)
    seg = ds.FSeg(a=ad, b=bd, y=y, sa=gu.dev_f32(sa), sb=gu.dev_f32(sb) if swiglu else None)
    (ds.ds_swiglu_l2_rows if swiglu else ds.ds_gate_l2_rows)([seg], eps)
    torch.cuda.synchronize()
    return gu.host_bits(y)


def check(swiglu, a, b, sa, sb, got, eps, flags=0, what=""):
    nt = oracle.default_threads()
    if swiglu:
        ref = oracle.swiglu_l2_rows(a, b, sa, sb, eps=eps, flags=flags, nthreads=nt)
        lo, hi = oracle.swiglu_l2_rows_interval(a, b, sa, sb, eps=eps, flags=flags, nthreads=nt)
    else:
        ref = oracle.gate_l2_rows(a, b, sa, eps=eps, flags=flags, nthreads=nt)
        lo, hi = oracle.gate_l2_rows_interval(a, b, sa, eps=eps, flags=flags, nthreads=nt)
    return gu.assert_bf16_rows(got, ref, lo, hi, what, ambiguous=gu.interval_admits_beyond_ulp(ref, lo, hi))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("swiglu", [False, True], ids=["gate", "swiglu"])
def test_tiny(path, swiglu):
    rng = np.random.default_rng(121)
    a, b, sa, sb = _inputs(rng, 32, 128)
    with ds.force_path(path):
        for eps in (1e-6, 0.0):
            got = run(swiglu, a, b, sa, sb, eps)
            check(swiglu, a, b, sa, sb, got, eps, what=f"tiny eps={eps}")


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("swiglu", [False, True], ids=["gate", "swiglu"])
def test_ragged_with_guards(path, swiglu):
    rng = np.random.default_rng(122)
    with ds.force_path(path):
        for cols in (1, 7, 8, 129, 1000, 4097, 8191, 16384):
            rows = 7
            ld = ((cols + 7) // 8) * 8 + 8
            a, b, sa, sb = _inputs(rng, rows, cols)
            bufs = []
            for src in (a, b):
                v, _ = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
                v.copy_(gu.dev_bf16(src))
                bufs.append(v)
            vecs = []
            for v in (sa, sb):   # NaN past cols: none of it may reach a row
                t = torch.full((cols + 8,), float("nan"), dtype=torch.float32, device="cuda")
                t[:cols].copy_(gu.dev_f32(v))
                vecs.append(t[:cols])
            y, ybuf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
            seg = ds.FSeg(a=bufs[0], b=bufs[1], y=y, sa=vecs[0], sb=vecs[1] if swiglu else None)
            (ds.ds_swiglu_l2_rows if swiglu else ds.ds_gate_l2_rows)([seg], 1e-6)
            torch.cuda.synchronize()
            assert gu.guards_intact(ybuf, rows, cols, ld, gu.CANARY_BF16), cols
            check(swiglu, a, b, sa, sb, gu.host_bits(y), 1e-6, what=f"cols={cols}")


@pytest.mark.parametrize("swiglu", [False, True], ids=["gate", "swiglu"])
def test_dory_widths_sampled(swiglu):
    rng = np.random.default_rng(123)
    for R, C in ((16384, 4096), (8192, 7168)):
        a, b, sa, sb = _inputs(rng, R, C)
        got = run(swiglu, a, b, sa, sb, 1e-6)
        rows = gu.sample_rows(R, 64, 124)
        check(swiglu, a[rows], b[rows], sa, sb, got[rows], 1e-6, what=f"[{R},{C}]")


def test_gate_fp32_exp_range():
    """Gate arguments below -88.7: fp32's exp(-z) overflows and the gate is
    exactly 0 (float64 keeps a tiny positive value); the interval holds it."""
    rng = np.random.default_rng(125)
    C = 512
    o = wl.normal_bf16(rng, (8, C))
    g = wl.to_bf16_bits(rng.uniform(-120.0, 4.0, (8, C)).astype(np.float32))
    sg = np.ones(C, np.float32)
    got = run(False, o, g, sg, sg, 0.0)
    check(False, o, g, sg, sg, got, 0.0, what="exp range")


def test_gate_halves_of_integers_exact():
    """The pages' gate 4: g = 0 makes every gated value half an integer,
    exact in fp32, so the sum is exact; the outputs equal the oracle's bits
    up to sqrt's and the division's last rounding (1 ulp)."""
    x = wl.integer_rows(126, 16, 4096)
    got = run(False, x, np.zeros_like(x), np.ones(4096, np.float32), None, 0.0)
    ref = oracle.gate_l2_rows(x, np.zeros_like(x), np.ones(4096, np.float32), eps=0.0)
    from tests.checks import bf16_ulp_violations
    assert not bf16_ulp_violations(got, ref).any()


@pytest.mark.parametrize("swiglu", [False, True], ids=["gate", "swiglu"])
def test_controls_are_detected(swiglu):
    """Each control drops one rounding point in the oracle; the GPU's rows
    must fall outside its interval somewhere."""
    rng = np.random.default_rng(127)
    a, b, sa, sb = _inputs(rng, 64, 1024)
    got = run(swiglu, a, b, sa, sb, 1e-6)
    check(swiglu, a, b, sa, sb, got, 1e-6)
    flags = [oracle.OR_DROP_SGATE, oracle.OR_DROP_SUP, oracle.OR_DROP_PRODUCT] if swiglu else [oracle.OR_DROP_GATED]
    nt = oracle.default_threads()
    for fl in flags:
        if swiglu:
            lo, hi = oracle.swiglu_l2_rows_interval(a, b, sa, sb, flags=fl, nthreads=nt)
        else:
            lo, hi = oracle.gate_l2_rows_interval(a, b, sa, flags=fl, nthreads=nt)
        assert bf16_interval_violations(got, lo, hi).any(), hex(fl)


@pytest.mark.parametrize("swiglu", [False, True], ids=["gate", "swiglu"])
def test_in_place(swiglu):
    rng = np.random.default_rng(128)
    a, b, sa, sb = _inputs(rng, 40, 1000)
    ref = run(swiglu, a, b, sa, sb, 1e-6)
    for target in ("a", "b"):
        ad, bd = gu.dev_bf16(a), gu.dev_bf16(b)
        y = ad if target == "a" else bd
        seg = ds.FSeg(a=ad, b=bd, y=y, sa=gu.dev_f32(sa), sb=gu.dev_f32(sb) if swiglu else None)
        (ds.ds_swiglu_l2_rows if swiglu else ds.ds_gate_l2_rows)([seg], 1e-6)
        torch.cuda.synchronize()
        assert np.array_equal(gu.host_bits(y), ref)


def test_fast_division_matches_ieee_on_every_fp32_input():
    """Markstein's reciprocal and quotient, where the rows use them, give
    the bits of IEEE division for every fp32 argument (2^32 of each)."""
    bad_r, bad_q, n_r, n_q = ds.ds_debug_division_check()
    assert bad_r == 0 and bad_q == 0, (bad_r, bad_q)
    # the fast range covers every argument above -87.3 (about 3.2e9 patterns
    # once the NaNs and those below are left out)
    assert n_r > 3_000_000_000 and n_q > 3_000_000_000, (n_r, n_q)


def test_negative_zero_and_tiny_gates():
    """-0, subnormal and +-inf entries in the scaled gate take the
    definition's value (silu(-0) = -0 and so on) with the rest of the unit."""
    C = 64
    g = np.zeros((4, C), np.uint16)
    g[0, ::2] = 0x8000                      # -0
    g[1, :] = 0x0001                        # smallest bf16 subnormal
    g[1, 1::2] = 0x8003
    g[2, :8] = 0x7F80                       # +inf: the unit takes IEEE division
    g[2, 8:] = wl.to_bf16_bits(np.linspace(-3, 3, C - 8).astype(np.float32))
    g[3, :] = wl.to_bf16_bits(np.linspace(-100, 100, C).astype(np.float32))
    u = wl.to_bf16_bits(np.ones((4, C), np.float32))
    one = np.ones(C, np.float32)
    for swiglu in (False, True):
        got = run(swiglu, u if not swiglu else g, g if not swiglu else u, one, one, 1e-6)
        a, b = (u, g) if not swiglu else (g, u)
        check(swiglu, a[[0, 1, 3]], b[[0, 1, 3]], one, one, got[[0, 1, 3]], 1e-6, what="special gates")
        if swiglu:   # silu(-0) = -0/2 = -0, kept through the product and the scaling
            assert np.all(got[0, ::2] == 0x8000) and np.all(got[0, 1::2] == 0)
