"""Every row class the planner picks on its own (DS_PATH_AUTO), compared with
the float64 oracle element by element.

The class of a row depends on (operation, cols) alone.  `AUTO_CASES` lists,
per operation, widths that land in each class the planner can pick (staged
slots of 16 to 112 KB, clusters of 2, 4 and 8 CTAs that each stage a slice
of the row, their partial sums meeting in distributed shared memory, the
two-pass stream); a
CPU test walks every width up to 140,000 columns and fails if a class has no
case here.  The GPU tests run each case with ragged column counts, padded
leading dimensions and canary guard rows, then check the cluster widths
for the two bit-exact invariants (TensorFold PR #1260: "a row's bits never
depend on the row count"; DragonScale, "Why scales drift": a row scaled by
2^k gives the same output at eps = 0).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from l2_row_b200 import ds
from l2_row_b200 import workloads as wl

W, C, T = ds.DS_PATH_WARP, ds.DS_PATH_CTA, ds.DS_PATH_CLUSTER
P2 = ds.DS_PATH_TWO_PASS

# (operation, cols, expected (path, threads per row, CTAs per row)); the
# activation backward and Dory cases run on dense matrices, so their widths
# keep rows 16-byte aligned (multiples of 8)
AUTO_CASES = {
    "fwd": [(768, (W, 32, 1)), (4100, (C, 64, 1)), (8200, (C, 128, 1)), (16390, (C, 256, 1)),
            (28680, (T, 128, 2)), (32768, (T, 128, 2)), (40001, (T, 128, 4)), (65536, (T, 128, 4)),
            (65541, (T, 128, 8)), (131072, (T, 128, 8)), (131077, (P2, 0, 8))],
    "bwd": [(1000, (W, 32, 1)), (3001, (C, 64, 1)), (6001, (C, 128, 1)), (12289, (C, 256, 1)),
            (16384, (T, 128, 2)), (20003, (T, 128, 4)), (32768, (T, 128, 4)), (50000, (T, 128, 8)),
            (65536, (T, 128, 8)), (65541, (P2, 0, 8))],
    "renorm": [(768, (W, 32, 1)), (4100, (C, 64, 1)), (8200, (C, 128, 1)), (16390, (C, 256, 1)),
               (30001, (T, 128, 2)), (50003, (T, 128, 4)), (100001, (T, 128, 8)), (131077, (P2, 0, 8))],
    "l2": [(1000, (W, 64, 1)), (6001, (C, 128, 1)), (12289, (C, 256, 1)), (16392, (T, 256, 2)),
           (24579, (T, 256, 2)), (40000, (T, 256, 4)), (65536, (T, 256, 4)), (65543, (T, 256, 8)),
           (131072, (T, 256, 8)), (131079, (P2, 0, 8))],
    "slerp": [(1000, (W, 64, 1)), (6001, (C, 128, 1)), (12289, (C, 256, 1)), (16392, (T, 256, 2)),
              (24579, (T, 256, 2)), (40000, (T, 256, 4)), (65536, (T, 256, 4)), (65543, (T, 256, 8)),
              (131072, (T, 256, 8)), (131079, (P2, 0, 8))],
    "project": [(1000, (W, 32, 1)), (3001, (C, 64, 1)), (6001, (C, 128, 1)), (12289, (C, 256, 1)),
                (16384, (T, 128, 2)), (20003, (T, 128, 4)), (50000, (T, 128, 8)), (65541, (P2, 0, 8))],
    "momentum": [(1000, (W, 32, 1)), (3001, (C, 64, 1)), (6001, (C, 128, 1)), (12289, (C, 256, 1)),
                 (16384, (T, 128, 2)), (20003, (T, 128, 4)), (50000, (T, 128, 8)), (65541, (P2, 0, 8))],
    "l2_bwd": [(1000, (W, 64, 1)), (4008, (C, 128, 1)), (10920, (C, 256, 1)), (10928, (T, 256, 2)),
               (16384, (T, 256, 2)), (30000, (T, 256, 4)), (50000, (T, 256, 8)), (87296, (T, 256, 8))],
    "slerp_bwd": [(1000, (W, 64, 1)), (4008, (C, 128, 1)), (10920, (C, 256, 1)), (10928, (T, 256, 2)),
                  (16384, (T, 256, 2)), (30000, (T, 256, 4)), (50000, (T, 256, 8)), (87296, (T, 256, 8))],
    "gate": [(1000, (W, 64, 1)), (7168, (C, 128, 1)), (16384, (C, 256, 1)), (16392, (T, 256, 2)),
             (40000, (T, 256, 4)), (100000, (T, 256, 8))],
    "swiglu": [(1000, (W, 64, 1)), (7168, (C, 128, 1)), (16384, (C, 256, 1)), (16392, (T, 256, 2)),
               (40000, (T, 256, 4)), (100000, (T, 256, 8))],
}
OPS = {"fwd": ds.DS_OP_WN_FORWARD, "bwd": ds.DS_OP_WN_BACKWARD, "renorm": ds.DS_OP_ROW_RENORM,
       "l2": ds.DS_OP_L2_ROWS, "slerp": ds.DS_OP_SLERP_ROWS, "project": ds.DS_OP_GRAD_PROJECT,
       "momentum": ds.DS_OP_RENORM_MOMENTUM, "l2_bwd": ds.DS_OP_L2_ROWS_BACKWARD,
       "slerp_bwd": ds.DS_OP_SLERP_ROWS_BACKWARD, "gate": ds.DS_OP_GATE_L2_ROWS,
       "swiglu": ds.DS_OP_SWIGLU_L2_ROWS}
CASE_IDS = [(op, cols) for op, cases in AUTO_CASES.items() for cols, _ in cases]


def row_class(op: str, cols: int):
    try:
        return ds.ds_row_class(OPS[op], cols)
    except ds.DSError:
        return None           # refused (longer than the operation's classes)


def test_every_auto_class_has_a_case():
    """Walk every width up to 140,000 columns (and a few beyond): each class
    the planner picks has a case above, and each case is in its class."""
    assert set(AUTO_CASES) == set(OPS)
    for op, cases in AUTO_CASES.items():
        picked = {row_class(op, c) for c in list(range(1, 140001)) + [262144, 1 << 20]}
        picked.discard(None)
        covered = {cls for _, cls in cases}
        assert picked == covered, (op, sorted(picked - covered), sorted(covered - picked))
        for cols, cls in cases:
            assert row_class(op, cols) == cls, (op, cols)


# ------------------------------------------------------------------ GPU --

def _ld(cols: int) -> int:
    return (cols + 7) // 8 * 8 + 8             # padded, 16-byte rows for fp32 and bf16


def _padded_copy(src: torch.Tensor, ld: int, canary):
    from tests import gpu_util as gu

    rows, cols = src.shape
    v, buf = gu.padded(rows, cols, ld, src.dtype, canary)
    v.copy_(src)
    return v, buf


def _weight_case(op: str, cols: int, rows: int, seed: int):
    from tests import gpu_util as gu

    rng = np.random.default_rng(seed)
    eps = 1e-6
    ld = _ld(cols)
    seg = wl.WeightSeg("w", wl.drifted_rows(rng, rows, cols, 0.02), wl.gains(rng, rows),
                       wl.normal_bf16(rng, (rows, cols), 1e-3))
    w, wbuf = _padded_copy(gu.dev_f32(seg.w), ld, gu.CANARY_F32)
    g = gu.dev_f32(seg.g)
    if op == "fwd":
        out, obuf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
        ds.ds_wn_forward([ds.WSeg(w=w, gain=g, w_eff=out)], "bf16", eps)
        torch.cuda.synchronize()
        assert gu.guards_intact(obuf, rows, cols, ld, gu.CANARY_BF16)
        gu.check_forward(seg, out, eps, "bf16", what=f"forward cols={cols}")
    elif op == "bwd":
        gy, _ = _padded_copy(gu.dev_bf16(seg.gy), ld, gu.CANARY_BF16)
        gw, gbuf = gu.padded(rows, cols, ld, torch.float32, gu.CANARY_F32)
        gg = torch.empty(rows, device="cuda")
        ds.ds_wn_backward([ds.WSeg(w=w, gain=g, gy=gy, grad_w=gw, grad_g=gg)], "bf16", eps)
        torch.cuda.synchronize()
        assert gu.guards_intact(gbuf, rows, cols, ld, gu.CANARY_F32)
        gu.check_backward(seg, gw, gg, eps, what=f"backward cols={cols}")
    elif op == "renorm":
        ds.ds_row_renorm([ds.WSeg(w=w)], eps)
        torch.cuda.synchronize()
        gu.check_renorm(seg, w, eps, what=f"renorm cols={cols}")
    else:
        st = wl.with_fp32_state([seg], seed + 1)[0]
        m, mbuf = _padded_copy(gu.dev_f32(st.gy), ld, gu.CANARY_F32)
        if op == "project":
            ds.ds_grad_project([ds.WSeg(w=w, grad_w=m)], eps)
            torch.cuda.synchronize()
            gu.check_project(st, m, eps, what=f"grad_project cols={cols}")
        else:
            ds.ds_renorm_momentum([ds.WSeg(w=w, grad_w=m)], eps)
            torch.cuda.synchronize()
            gu.check_momentum(st, w, m, eps, what=f"renorm_momentum cols={cols}")
        assert gu.guards_intact(mbuf, rows, cols, ld, gu.CANARY_F32)
    assert gu.guards_intact(wbuf, rows, cols, ld, gu.CANARY_F32)


def _act_case(op: str, cols: int, rows: int, seed: int):
    from tests import gpu_util as gu

    rng = np.random.default_rng(seed)
    eps = 1e-6
    ld = _ld(cols)
    act = wl.ActRows("a", wl.normal_bf16(rng, (rows, cols)), wl.normal_bf16(rng, (rows, cols)),
                     wl.alpha_vec(rng, cols))
    x, _ = _padded_copy(gu.dev_bf16(act.x), ld, gu.CANARY_BF16)
    r, _ = _padded_copy(gu.dev_bf16(act.r), ld, gu.CANARY_BF16)
    y, ybuf = gu.padded(rows, cols, ld, torch.bfloat16, gu.CANARY_BF16)
    if op == "l2":
        for res in (False, True):
            ds.ds_l2_rows([ds.ASeg(x=x, r=r if res else None, y=y)], eps)
            torch.cuda.synchronize()
            assert gu.guards_intact(ybuf, rows, cols, ld, gu.CANARY_BF16)
            gu.check_l2(act, y, eps, residual=res, what=f"l2 residual={res} cols={cols}")
    else:
        ds.ds_slerp_rows([ds.ASeg(x=x, r=r, y=y, alpha=gu.dev_f32(act.alpha))], eps)
        torch.cuda.synchronize()
        assert gu.guards_intact(ybuf, rows, cols, ld, gu.CANARY_BF16)
        gu.check_slerp(act, y, eps, what=f"slerp cols={cols}")


def _act_bwd_case(op: str, cols: int, rows: int, seed: int):
    from tests import test_parity_act_bwd as ab

    rng = np.random.default_rng(seed)
    x, r, dy = (wl.normal_bf16(rng, (rows, cols)) for _ in range(3))
    if op == "l2_bwd":
        for rr in (None, r):
            got = ab.run_l2_bwd(x, rr, dy, 1e-6)
            ab.check_l2_bwd(x, rr, dy, got, 1e-6, what=f"l2 bwd residual={rr is not None} cols={cols}")
    else:
        alpha = wl.alpha_vec(rng, cols)
        got = ab.run_slerp_bwd(x, r, alpha, dy, 1e-6)
        ab.check_slerp_bwd(x, r, alpha, dy, got, 1e-6, strict=False, what=f"slerp bwd cols={cols}")


def _fused_case(op: str, cols: int, rows: int, seed: int):
    from tests import test_parity_fused as fu

    rng = np.random.default_rng(seed)
    a, b, sa, sb = fu._inputs(rng, rows, cols)
    swiglu = op == "swiglu"
    got = fu.run(swiglu, a, b, sa, sb, 1e-6)
    fu.check(swiglu, a, b, sa, sb, got, 1e-6, what=f"{op} cols={cols}")


@pytest.mark.gpu
@pytest.mark.parametrize("op,cols", CASE_IDS, ids=[f"{o}-{c}" for o, c in CASE_IDS])
def test_auto_class_matches_oracle(op, cols):
    expected = dict(AUTO_CASES[op])[cols]
    assert row_class(op, cols) == expected
    rows = 5 if cols > 16384 else 9
    seed = 1000 + cols
    if op in ("fwd", "bwd", "renorm", "project", "momentum"):
        _weight_case(op, cols, rows, seed)
    elif op in ("l2", "slerp"):
        _act_case(op, cols, rows, seed)
    elif op in ("l2_bwd", "slerp_bwd"):
        _act_bwd_case(op, cols, rows, seed)
    else:
        _fused_case(op, cols, rows, seed)
    assert ds.ds_get_device_status() == ds.DS_OK


CLUSTER_WIDTHS = {"fwd": [30001, 40001, 100001], "bwd": [16384, 20003, 50000], "l2": [24579, 40000, 100000],
                  "slerp": [24579, 40000, 100000]}


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.gpu
@pytest.mark.parametrize("op", list(CLUSTER_WIDTHS))
def test_cluster_rows_count_invariance(op):
    """Each row alone, in the full launch and split over several segments of
    one call gives the same bits."""
    from tests import gpu_util as gu

    rng = np.random.default_rng(71)
    eps = 1e-6
    for cols in CLUSTER_WIDTHS[op]:
        R = 7
        ld = _ld(cols)

        def pad(t, canary):
            return _padded_copy(t, ld, canary)[0]

        def empty(dt):
            return gu.padded(R, cols, ld, dt, gu.CANARY_BF16 if dt == torch.bfloat16 else gu.CANARY_F32)[0]

        if op in ("fwd", "bwd"):
            w = pad(gu.dev_f32(wl.drifted_rows(rng, R, cols, 0.02)), gu.CANARY_F32)
            g = gu.dev_f32(wl.gains(rng, R))
            gy = pad(gu.dev_bf16(wl.normal_bf16(rng, (R, cols), 1e-3)), gu.CANARY_BF16)

            def call(lo, hi, out, gout=None):
                if op == "fwd":
                    return ds.WSeg(w=w[lo:hi], gain=g[lo:hi], w_eff=out[lo:hi])
                return ds.WSeg(w=w[lo:hi], gain=g[lo:hi], gy=gy[lo:hi], grad_w=out[lo:hi], grad_g=gout[lo:hi])

            dt = torch.bfloat16 if op == "fwd" else torch.float32
            fn = (lambda segs: ds.ds_wn_forward(segs, "bf16", eps)) if op == "fwd" else \
                 (lambda segs: ds.ds_wn_backward(segs, "bf16", eps))
        else:
            x = pad(gu.dev_bf16(wl.normal_bf16(rng, (R, cols))), gu.CANARY_BF16)
            r = pad(gu.dev_bf16(wl.normal_bf16(rng, (R, cols))), gu.CANARY_BF16)
            al = gu.dev_f32(wl.alpha_vec(rng, cols))

            def call(lo, hi, out, gout=None):
                return ds.ASeg(x=x[lo:hi], r=r[lo:hi], y=out[lo:hi], alpha=al if op == "slerp" else None)

            dt = torch.bfloat16
            fn = (lambda segs: ds.ds_slerp_rows(segs, eps)) if op == "slerp" else \
                 (lambda segs: ds.ds_l2_rows(segs, eps))
        full = empty(dt)
        gfull = torch.empty(R, device="cuda")
        fn([call(0, R, full, gfull)])
        parts = empty(dt)
        gparts = torch.empty_like(gfull)
        cuts = [0, 1, 3, 4, 7]
        fn([call(a, b, parts, gparts) for a, b in zip(cuts, cuts[1:])])
        for k in (0, 4, 6):
            one = empty(dt)
            gone = torch.empty_like(gfull)
            fn([call(k, k + 1, one, gone)])
            torch.cuda.synchronize()
            assert torch.equal(_bits(one[k]), _bits(full[k])), (op, cols, k)
            if op == "bwd":
                assert torch.equal(gone[k], gfull[k])
        torch.cuda.synchronize()
        assert torch.equal(_bits(parts), _bits(full)), (op, cols)
        if op == "bwd":
            assert torch.equal(gparts, gfull)


@pytest.mark.gpu
def test_cluster_rows_power_of_two_scale_invariance():
    """At eps = 0 a row scaled by 2^k (exact in fp32) gives the same bits,
    also where the scaled sum of squares leaves fp32's range and the rows
    are re-summed after an exact rescale."""
    from tests import gpu_util as gu

    rng = np.random.default_rng(72)
    for cols in (30004, 40004, 100004):       # dense fp32 rows: multiples of 4
        w = wl.drifted_rows(rng, 3, cols, 1.0)
        base = gu.run_forward([wl.WeightSeg("w", w, None, None)], "f32", 0.0)[0]
        for k in (-70, -20, 20, 70):
            ws = np.ldexp(w, k).astype(np.float32)
            assert np.array_equal(np.ldexp(ws, -k), w)
            got = gu.run_forward([wl.WeightSeg("w", ws, None, None)], "f32", 0.0)[0]
            assert torch.equal(got, base), (cols, k)
    for cols in (24584, 40000, 100000):       # dense bf16 rows: multiples of 8
        xf = wl.bf16_bits_to_f32(wl.normal_bf16(rng, (3, cols)))
        ybase = gu.run_l2([wl.ActRows("x", wl.to_bf16_bits(xf), None)], 0.0, residual=False)[0]
        for k in (-60, -20, 20, 60):
            xs = np.ldexp(xf, k).astype(np.float32)
            assert np.array_equal(wl.bf16_bits_to_f32(wl.to_bf16_bits(xs)), xs)
            y = gu.run_l2([wl.ActRows("x", wl.to_bf16_bits(xs), None)], 0.0, residual=False)[0]
            assert torch.equal(_bits(y), _bits(ybase)), (cols, k)
