"""The C ABI without a GPU: the library loads, exports every symbol
include/ds.h declares, plans row classes from (op, cols) alone, and rejects
bad arguments on the host before any launch (no kernel runs here)."""
from __future__ import annotations

import ctypes as ct
import os
import re

import pytest

from l2_row_b200 import ds

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions() -> set[str]:
    src = open(os.path.join(ROOT, "include", "ds.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(ds_[a-z_0-9]+)\s*\(", src))


def test_every_declared_symbol_is_exported():
    decl = declared_functions()
    assert decl == set(ds.EXPORTS)
    for name in decl:
        assert hasattr(ds.lib(), name), name


def test_status_strings_and_version():
    for code in range(8):
        assert ds.ds_status_string(code) not in ("", "unknown status")
    assert ds.ds_status_string(99) == "unknown status"
    assert ds.ds_version() >= 100


# ------------------------------------------------------------- row classes --

W_OPS = (ds.DS_OP_WN_FORWARD, ds.DS_OP_WN_BACKWARD, ds.DS_OP_ROW_RENORM, ds.DS_OP_GRAD_PROJECT,
         ds.DS_OP_RENORM_MOMENTUM)
A_OPS = (ds.DS_OP_L2_ROWS, ds.DS_OP_SLERP_ROWS)


@pytest.mark.parametrize("op,cols,want", [
    (ds.DS_OP_WN_FORWARD, 768, (ds.DS_PATH_WARP, 32, 1)),     # staged rows <= 16 KB: warp per row
    (ds.DS_OP_WN_FORWARD, 2048, (ds.DS_PATH_WARP, 32, 1)),
    (ds.DS_OP_WN_BACKWARD, 768, (ds.DS_PATH_WARP, 32, 1)),
    (ds.DS_OP_WN_BACKWARD, 2048, (ds.DS_PATH_WARP, 32, 1)),   # w + fp32 GY = 16 KB
    (ds.DS_OP_WN_BACKWARD, 2049, (ds.DS_PATH_CTA, 64, 1)),   # w + fp32 GY > 16 KB: 32 KB slots, 2 warps
    (ds.DS_OP_ROW_RENORM, 128, (ds.DS_PATH_WARP, 32, 1)),
    (ds.DS_OP_L2_ROWS, 4096, (ds.DS_PATH_WARP, 64, 1)),       # x + r = 16 KB, a pair of warps
    (ds.DS_OP_SLERP_ROWS, 7168, (ds.DS_PATH_CTA, 128, 1)),    # 28 KB: 32 KB slots, 4 warps
    (ds.DS_OP_L2_ROWS, 16384, (ds.DS_PATH_CTA, 256, 1)),      # 64 KB slots, 8 warps
    (ds.DS_OP_WN_FORWARD, 14336, (ds.DS_PATH_CTA, 128, 1)),   # 56 KB: 64 KB slots, 4 warps
    (ds.DS_OP_WN_BACKWARD, 14336, (ds.DS_PATH_CTA, 256, 1)),  # 112 KB (fp32 GY layout): 112 KB slots, 8 warps
    (ds.DS_OP_WN_BACKWARD, 14337, (ds.DS_PATH_CLUSTER, 128, 2)),   # two 56 KB slices: 64 KB slots
    (ds.DS_OP_WN_FORWARD, 131072, (ds.DS_PATH_CLUSTER, 128, 8)),   # eight 64 KB slices
    (ds.DS_OP_WN_FORWARD, 131073, (ds.DS_PATH_TWO_PASS, 0, 8)),
    (ds.DS_OP_GRAD_PROJECT, 2048, (ds.DS_PATH_WARP, 32, 1)),  # w + G fp32 = 16 KB
    (ds.DS_OP_RENORM_MOMENTUM, 2049, (ds.DS_PATH_CTA, 64, 1)),
    (ds.DS_OP_GRAD_PROJECT, 14336, (ds.DS_PATH_CTA, 256, 1)),
    (ds.DS_OP_GRAD_PROJECT, 16384, (ds.DS_PATH_CLUSTER, 128, 2)),
    (ds.DS_OP_RENORM_MOMENTUM, 65537, (ds.DS_PATH_TWO_PASS, 0, 8)),
    (ds.DS_OP_SLERP_ROWS, 16385, (ds.DS_PATH_CLUSTER, 256, 2)),
    (ds.DS_OP_L2_ROWS_BACKWARD, 16384, (ds.DS_PATH_CLUSTER, 256, 2)),  # x, r, dy: 96 KB in two slices
    (ds.DS_OP_SWIGLU_L2_ROWS, 131072, (ds.DS_PATH_CLUSTER, 256, 8)),
    (ds.DS_OP_SLERP_ROWS, 262144, (ds.DS_PATH_TWO_PASS, 0, 8)),
])
def test_row_class_for_workload_shapes(op, cols, want):
    assert ds.ds_row_class(op, cols) == want


def test_row_class_is_monotone_and_fits():
    """Staged classes take rows by their staged bytes: one CTA per row in the
    smallest slot of 16, 32 or 64 KB (112 KB for weights) that holds the row;
    longer rows are split over the smallest cluster of 2, 4 or 8 CTAs whose
    slices (units rounded up to an even count) fit 64 KB, in the smallest
    slot that holds a slice; then the two-pass class.  The class never
    shrinks as rows grow."""
    order = {ds.DS_PATH_WARP: 0, ds.DS_PATH_CTA: 1, ds.DS_PATH_CLUSTER: 2, ds.DS_PATH_TWO_PASS: 3}
    for op in W_OPS + A_OPS:
        e = 4 if op in W_OPS else 8
        base = 1 if op in W_OPS else 2
        ub = 16 if op in (ds.DS_OP_WN_FORWARD, ds.DS_OP_ROW_RENORM) else 32
        prev = (0, 0, 0)
        for cols in sorted(set(list(range(1, 600, 7)) + [2 ** k + d for k in range(9, 19) for d in (-1, 0, 1)])):
            path, g, cl = ds.ds_row_class(op, cols)
            nu = -(-cols // e)
            staged = ub * nu

            def slice_bytes(n):
                return ub * ((-(-nu // n) + 1) // 2 * 2)

            if path == ds.DS_PATH_WARP:
                assert staged <= 16384 and g == 32 * base and cl == 1
            elif path == ds.DS_PATH_CTA:
                top = 114688 if op in W_OPS else 65536
                slot = next(x for x in (32768, 65536, 114688) if staged <= x)
                warps = 8 if slot == 114688 else base * slot // 16384
                assert 16384 < staged <= top and g == 32 * warps and cl == 1
            elif path == ds.DS_PATH_CLUSTER:
                top = 114688 if op in W_OPS else 65536
                assert staged > top and cl in (2, 4, 8)
                assert slice_bytes(cl) <= 65536 and (cl == 2 or slice_bytes(cl // 2) > 65536)
                slot = next(x for x in (16384, 32768, 65536) if slice_bytes(cl) <= x)
                assert g == 32 * base * slot // 16384
            else:
                assert slice_bytes(8) > 65536
            key = (order[path], cl)
            assert key >= prev, (op, cols)
            prev = key


def test_forced_paths():
    with ds.force_path(ds.DS_PATH_TWO_PASS):
        assert ds.ds_row_class(ds.DS_OP_L2_ROWS, 128)[0] == ds.DS_PATH_TWO_PASS
    with ds.force_path(ds.DS_PATH_CLUSTER):       # two 1.5 KB slices in 16 KB slots
        assert ds.ds_row_class(ds.DS_OP_WN_FORWARD, 768) == (ds.DS_PATH_CLUSTER, 32, 2)
    with ds.force_path(ds.DS_PATH_WARP):  # does not fit: automatic choice
        assert ds.ds_row_class(ds.DS_OP_L2_ROWS, 8192)[0] == ds.DS_PATH_CTA
    with ds.force_path(ds.DS_PATH_CTA):
        assert ds.ds_row_class(ds.DS_OP_WN_FORWARD, 128) == (ds.DS_PATH_CTA, 64, 1)
    assert ds.ds_row_class(ds.DS_OP_L2_ROWS, 128)[0] == ds.DS_PATH_WARP
    with pytest.raises(ds.DSError):
        ds.ds_debug_force_path(9)


# ------------------------------------------------------ host-side validation --
# Fake, never dereferenced device addresses: every call below fails on the
# host before anything is launched.

BASE = 0x7F0000000000


def wseg(**kw):
    d = dict(w=BASE, gain=0, w_eff=BASE + (1 << 30), gy=BASE + (2 << 30), grad_w=BASE + (3 << 30),
             grad_g=0, rows=4, cols=8, ld=8, ld_out=8, radius=1.0)
    d.update(kw)
    return ds.ds_wseg(**d)


def aseg(**kw):
    d = dict(x=BASE, r=0, y=BASE + (1 << 30), alpha=BASE + (2 << 30), rows=4, cols=8, ld=8)
    d.update(kw)
    return ds.ds_aseg(**d)


NO_DTYPE = ("ds_row_renorm", "ds_grad_project", "ds_renorm_momentum")


def call_w(fn, segs, dt=ds.DS_BF16, eps=1e-6):
    arr = (ds.ds_wseg * max(1, len(segs)))(*segs)
    if fn in NO_DTYPE:
        return getattr(ds.lib(), fn)(arr, len(segs), ct.c_float(eps), None)
    return getattr(ds.lib(), fn)(arr, len(segs), dt, ct.c_float(eps), None)


def call_a(fn, segs, eps=1e-6):
    arr = (ds.ds_aseg * max(1, len(segs)))(*segs)
    return getattr(ds.lib(), fn)(arr, len(segs), ct.c_float(eps), None)


@pytest.mark.parametrize("fn", ["ds_wn_forward", "ds_wn_backward", "ds_row_renorm", "ds_grad_project",
                                "ds_renorm_momentum"])
def test_weight_validation(fn):
    E = ds
    before = ds.ds_launch_count()
    assert call_w(fn, [wseg(rows=-1)]) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg(cols=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg(ld=4)]) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg(w=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg(w=BASE + 4)]) == E.DS_ERR_ALIGNMENT
    assert call_w(fn, [wseg(ld=10, cols=8)]) == E.DS_ERR_ALIGNMENT          # 40-byte rows
    assert call_w(fn, [wseg()], eps=-1.0) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg()], eps=float("nan")) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg()], eps=float("inf")) == E.DS_ERR_INVALID_ARG
    assert call_w(fn, [wseg(radius=float("nan"))]) == E.DS_ERR_INVALID_ARG
    arr = (ds.ds_wseg * 1)(wseg())
    if fn in NO_DTYPE:
        assert getattr(ds.lib(), fn)(None, 1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
        assert getattr(ds.lib(), fn)(arr, -1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
        assert getattr(ds.lib(), fn)(arr, E.DS_MAX_SEGMENTS + 1, ct.c_float(1e-6), None) == \
            E.DS_ERR_TOO_MANY_SEGMENTS
    else:
        assert call_w(fn, [wseg()], dt=7) == E.DS_ERR_UNSUPPORTED_DTYPE
        assert call_w(fn, [wseg(ld_out=4)]) == E.DS_ERR_INVALID_ARG
    # empty work launches nothing and succeeds without touching the device
    assert call_w(fn, []) == E.DS_OK
    assert call_w(fn, [wseg(rows=0, w=0, w_eff=0, gy=0, grad_w=0)]) == E.DS_OK
    assert ds.ds_launch_count() == before
    assert "segment 0" in ds.ds_last_error() or ds.ds_last_error() == ""


def test_weight_specific_validation():
    E = ds
    assert call_w("ds_wn_forward", [wseg(w_eff=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_forward", [wseg(w_eff=BASE + (1 << 30) + 8)]) == E.DS_ERR_ALIGNMENT
    assert call_w("ds_wn_backward", [wseg(gy=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_backward", [wseg(grad_w=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_backward", [wseg(gain=BASE + (4 << 30), grad_g=0)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_backward", [wseg(gain=BASE + (4 << 30) + 2, grad_g=BASE + (5 << 30))]) == \
        E.DS_ERR_ALIGNMENT
    # bf16 W_eff rows need ld_out % 8 == 0; fp32 rows need ld_out % 4 == 0
    assert call_w("ds_wn_forward", [wseg(ld_out=12, ld=12)]) == E.DS_ERR_ALIGNMENT
    assert ds.ds_last_error().startswith("segment 0")


def test_optimizer_call_validation():
    E = ds
    for fn in ("ds_grad_project", "ds_renorm_momentum"):
        # grad_w holds the gradient / momentum: required, aligned, w's ld
        assert call_w(fn, [wseg(grad_w=0)]) == E.DS_ERR_INVALID_ARG
        assert call_w(fn, [wseg(grad_w=BASE + (3 << 30) + 4)]) == E.DS_ERR_ALIGNMENT
        # gy, w_eff, gain, ld_out are not read: their values do not matter
        before = ds.ds_launch_count()
        assert call_w(fn, [wseg(gy=0, w_eff=0, ld_out=0, rows=0)]) == E.DS_OK
        assert ds.ds_launch_count() == before
        # the buffer must not overlap w (it is updated in place)
        assert call_w(fn, [wseg(grad_w=BASE)]) == E.DS_ERR_OVERLAP
        assert call_w(fn, [wseg(grad_w=BASE + 64)]) == E.DS_ERR_OVERLAP
        # two segments updating the same gradient rows
        assert call_w(fn, [wseg(), wseg(w=BASE + (8 << 30))]) == E.DS_ERR_OVERLAP


def test_weight_overlap_rejected():
    E = ds
    # W_eff over w
    assert call_w("ds_wn_forward", [wseg(w_eff=BASE + 16)], dt=ds.DS_F32) == E.DS_ERR_OVERLAP
    # grad_w over gy, even exactly
    assert call_w("ds_wn_backward", [wseg(grad_w=BASE + (2 << 30))], dt=ds.DS_F32) == E.DS_ERR_OVERLAP
    # two segments writing the same rows
    a = wseg()
    b = wseg(w=BASE + (8 << 30))
    assert call_w("ds_wn_forward", [a, b]) == E.DS_ERR_OVERLAP
    # renorm of two overlapping segments
    assert call_w("ds_row_renorm", [wseg(), wseg(w=BASE + 64)]) == E.DS_ERR_OVERLAP
    # backward grad_g overlapping the gain vector
    assert call_w("ds_wn_backward", [wseg(gain=BASE + (4 << 30), grad_g=BASE + (4 << 30) + 4)]) == \
        E.DS_ERR_OVERLAP


@pytest.mark.parametrize("fn", ["ds_l2_rows", "ds_slerp_rows"])
def test_activation_validation(fn):
    E = ds
    slerp = fn == "ds_slerp_rows"
    r = BASE + (3 << 30)
    good = dict(r=r) if slerp else {}
    assert call_a(fn, [aseg(rows=-1, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_a(fn, [aseg(cols=0, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_a(fn, [aseg(ld=7, cols=8, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_a(fn, [aseg(ld=12, cols=8, **good)]) == E.DS_ERR_ALIGNMENT   # 24-byte bf16 rows
    assert call_a(fn, [aseg(x=0, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_a(fn, [aseg(y=0, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_a(fn, [aseg(x=BASE + 2, **good)]) == E.DS_ERR_ALIGNMENT
    assert call_a(fn, [aseg(**good)], eps=-1e-6) == E.DS_ERR_INVALID_ARG
    # partial overlap of y with x is refused (exact aliasing is allowed: tested on the GPU)
    assert call_a(fn, [aseg(y=BASE + 16, **good)]) == E.DS_ERR_OVERLAP
    assert call_a(fn, [aseg(**good), aseg(x=BASE + (6 << 30), y=BASE + (1 << 30) + 16, **good)]) == \
        E.DS_ERR_OVERLAP
    if slerp:
        assert call_a(fn, [aseg()]) == E.DS_ERR_INVALID_ARG                # out is required
        assert call_a(fn, [aseg(r=r, alpha=0)]) == E.DS_ERR_INVALID_ARG
        assert call_a(fn, [aseg(r=r, alpha=BASE + (2 << 30) + 4)]) == E.DS_ERR_ALIGNMENT
    else:
        assert call_a(fn, [aseg(r=BASE + 2)]) == E.DS_ERR_ALIGNMENT
    assert call_a(fn, []) == E.DS_OK
    assert call_a(fn, [aseg(rows=0, x=0, y=0, alpha=0)]) == E.DS_OK


def test_binding_marshals_tensors_and_rejects_bad_views():
    import torch

    w = torch.zeros(4, 8)
    seg = ds.WSeg(w=w, w_eff=torch.zeros(4, 8, dtype=torch.bfloat16))
    c = seg.to_c()
    assert (c.rows, c.cols, c.ld, c.ld_out) == (4, 8, 8, 8)
    wide = torch.zeros(4, 16)
    c = ds.WSeg(w=wide[:, :8], w_eff=torch.zeros(4, 8)).to_c()
    assert (c.ld, c.cols) == (16, 8)
    with pytest.raises(ValueError):
        ds.WSeg(w=w, w_eff=torch.zeros(3, 8)).to_c()
    with pytest.raises(ValueError):
        ds.WSeg(w=w.t().contiguous().t(), w_eff=torch.zeros(4, 8)).to_c()
    a = ds.ASeg(x=torch.zeros(2, 16, dtype=torch.bfloat16), y=torch.zeros(2, 16, dtype=torch.bfloat16)).to_c()
    assert (a.rows, a.cols, a.ld, a.r) == (2, 16, 16, None)


def test_binding_accepts_empty_tensors_with_any_strides():
    import torch

    w = torch.zeros(64, 0).t()          # shape (0, 64), stride (1, 0)
    c = ds.WSeg(w=w, w_eff=torch.zeros(0, 64)).to_c()
    assert (c.rows, c.cols) == (0, 64)


# ------------------------------------------------- activation backward calls --

def agseg(**kw):
    d = dict(x=BASE, r=0, dy=BASE + (1 << 30), dx=BASE + (2 << 30), dr=BASE + (3 << 30),
             alpha=BASE + (4 << 30), rows=4, cols=8, ld=8, ld_d=8)
    d.update(kw)
    return ds.ds_agseg(**d)


def call_g(fn, segs, eps=1e-6, dalpha=0, ws=0, ws_bytes=0):
    arr = (ds.ds_agseg * max(1, len(segs)))(*segs)
    lib = ds.lib()
    if fn == "ds_l2_rows_backward":
        return lib.ds_l2_rows_backward(arr, len(segs), ct.c_float(eps), None)
    return lib.ds_slerp_rows_backward(arr, len(segs), ct.c_float(eps), dalpha, ws, ws_bytes, None)


def test_backward_row_classes():
    # x, r, dy staged: 48 bytes per 8 columns, at most 64 KB
    assert ds.ds_row_class(ds.DS_OP_L2_ROWS_BACKWARD, 2728) == (ds.DS_PATH_WARP, 64, 1)
    assert ds.ds_row_class(ds.DS_OP_SLERP_ROWS_BACKWARD, 4096) == (ds.DS_PATH_CTA, 128, 1)
    assert ds.ds_row_class(ds.DS_OP_SLERP_ROWS_BACKWARD, 7168) == (ds.DS_PATH_CTA, 256, 1)
    assert ds.ds_row_class(ds.DS_OP_L2_ROWS_BACKWARD, 10920)[0] == ds.DS_PATH_CTA
    # longer rows: 2, 4 or 8 CTAs, each staging a slice of at most 64 KB
    assert ds.ds_row_class(ds.DS_OP_L2_ROWS_BACKWARD, 10921) == (ds.DS_PATH_CLUSTER, 256, 2)
    assert ds.ds_row_class(ds.DS_OP_SLERP_ROWS_BACKWARD, 16384) == (ds.DS_PATH_CLUSTER, 256, 2)
    assert ds.ds_row_class(ds.DS_OP_SLERP_ROWS_BACKWARD, 87296) == (ds.DS_PATH_CLUSTER, 256, 8)
    with pytest.raises(ds.DSError):
        ds.ds_row_class(ds.DS_OP_L2_ROWS_BACKWARD, 87297)
    with ds.force_path(ds.DS_PATH_TWO_PASS):   # no two-pass class: the staged one is kept
        assert ds.ds_row_class(ds.DS_OP_L2_ROWS_BACKWARD, 128)[0] == ds.DS_PATH_WARP


@pytest.mark.parametrize("fn", ["ds_l2_rows_backward", "ds_slerp_rows_backward"])
def test_backward_validation(fn):
    E = ds
    slerp = fn == "ds_slerp_rows_backward"
    good = dict(r=BASE + (5 << 30)) if slerp else {}
    before = ds.ds_launch_count()
    assert call_g(fn, [agseg(rows=-1, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_g(fn, [agseg(ld_d=4, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_g(fn, [agseg(dx=0, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_g(fn, [agseg(dy=0, **good)]) == E.DS_ERR_INVALID_ARG
    assert call_g(fn, [agseg(dx=BASE + (2 << 30) + 4, **good)]) == E.DS_ERR_ALIGNMENT
    if slerp:   # x, r, dy staged in 8 slices of 64 KB: 87,296 columns at most
        assert call_g(fn, [agseg(cols=87297, ld=87304, ld_d=87300, **good)]) == E.DS_ERR_INVALID_ARG
    else:       # without a residual x and dy: 131,072 columns; with one 87,296
        assert call_g(fn, [agseg(cols=131073, ld=131080, ld_d=131076)]) == E.DS_ERR_INVALID_ARG
        assert call_g(fn, [agseg(cols=87297, ld=87304, ld_d=87300, r=BASE + (5 << 30))]) == E.DS_ERR_INVALID_ARG
    # dx over an input
    assert call_g(fn, [agseg(dx=BASE + (1 << 30), **good)]) == E.DS_ERR_OVERLAP
    assert call_g(fn, [agseg(rows=0, x=0, dy=0, dx=0, dr=0, **good)]) == E.DS_OK
    if slerp:
        assert call_g(fn, [agseg()]) == E.DS_ERR_INVALID_ARG                 # out (r) required
        assert call_g(fn, [agseg(dr=0, **good)]) == E.DS_ERR_INVALID_ARG
        assert call_g(fn, [agseg(alpha=0, **good)]) == E.DS_ERR_INVALID_ARG
        assert call_g(fn, [agseg(dr=BASE + (2 << 30), **good)]) == E.DS_ERR_OVERLAP   # dr over dx
        need = ds.ds_slerp_rows_backward_workspace(8)
        assert need > 0 and ds.ds_slerp_rows_backward_workspace(0) == 0
        da, ws = BASE + (6 << 30), BASE + (7 << 30)
        assert call_g(fn, [agseg(**good)], dalpha=da) == E.DS_ERR_INVALID_ARG          # no workspace
        assert call_g(fn, [agseg(**good)], dalpha=da, ws=ws + 16, ws_bytes=need) == E.DS_ERR_ALIGNMENT
        assert call_g(fn, [agseg(**good)], dalpha=da, ws=ws, ws_bytes=need - 1) == E.DS_ERR_INVALID_ARG
        other = agseg(x=BASE + (8 << 30), r=BASE + (9 << 30), dy=BASE + (10 << 30), dx=BASE + (11 << 30),
                      dr=BASE + (12 << 30), alpha=BASE + (13 << 30))
        assert call_g(fn, [agseg(**good), other], dalpha=da, ws=ws, ws_bytes=need) == E.DS_ERR_INVALID_ARG
        assert call_g(fn, [agseg(**good)], dalpha=ws, ws=ws, ws_bytes=need) == E.DS_ERR_OVERLAP
    assert ds.ds_launch_count() == before


# ----------------------------------------------------------- Dory's rows --

def fseg(**kw):
    d = dict(a=BASE, b=BASE + (1 << 30), y=BASE + (2 << 30), sa=BASE + (3 << 30), sb=BASE + (4 << 30),
             rows=4, cols=8, ld=8)
    d.update(kw)
    return ds.ds_fseg(**d)


def call_f(fn, segs, eps=1e-6):
    arr = (ds.ds_fseg * max(1, len(segs)))(*segs)
    return getattr(ds.lib(), fn)(arr, len(segs), ct.c_float(eps), None)


def test_fused_row_classes():
    # a and b staged: 32 bytes per 8 columns; a pair of warps per 16 KB of slot
    assert ds.ds_row_class(ds.DS_OP_GATE_L2_ROWS, 4096) == (ds.DS_PATH_WARP, 64, 1)
    assert ds.ds_row_class(ds.DS_OP_SWIGLU_L2_ROWS, 7168) == (ds.DS_PATH_CTA, 128, 1)
    assert ds.ds_row_class(ds.DS_OP_SWIGLU_L2_ROWS, 16384) == (ds.DS_PATH_CTA, 256, 1)
    assert ds.ds_row_class(ds.DS_OP_GATE_L2_ROWS, 16385) == (ds.DS_PATH_CLUSTER, 256, 2)
    assert ds.ds_row_class(ds.DS_OP_GATE_L2_ROWS, 131072) == (ds.DS_PATH_CLUSTER, 256, 8)
    with pytest.raises(ds.DSError):
        ds.ds_row_class(ds.DS_OP_GATE_L2_ROWS, 131073)


@pytest.mark.parametrize("fn", ["ds_gate_l2_rows", "ds_swiglu_l2_rows"])
def test_fused_validation(fn):
    E = ds
    before = ds.ds_launch_count()
    assert call_f(fn, [fseg(rows=-1)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(a=0)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(b=0)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(y=0)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(sa=0)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(sa=BASE + (3 << 30) + 4)]) == E.DS_ERR_ALIGNMENT
    assert call_f(fn, [fseg(a=BASE + 2)]) == E.DS_ERR_ALIGNMENT
    assert call_f(fn, [fseg(cols=131073, ld=131080)]) == E.DS_ERR_INVALID_ARG   # past 8 slices of 64 KB
    assert call_f(fn, [fseg(y=BASE + 16)]) == E.DS_ERR_OVERLAP            # partial overlap with a
    assert call_f(fn, [fseg()], eps=-1.0) == E.DS_ERR_INVALID_ARG
    if fn == "ds_swiglu_l2_rows":
        assert call_f(fn, [fseg(sb=0)]) == E.DS_ERR_INVALID_ARG
    assert call_f(fn, [fseg(rows=0, a=0, b=0, y=0)]) == E.DS_OK
    assert ds.ds_launch_count() == before


# ------------------------------------------------------- Dory's q/k rows --

def qkseg(**kw):
    d = dict(q=BASE, k=BASE + (1 << 30), v=BASE + (2 << 30), q_out=BASE + (3 << 30), k_cache=BASE + (4 << 30),
             v_cache=BASE + (5 << 30), pos=BASE + (6 << 30), slot=None, inv_freq=BASE + (6 << 30) + 4096,
             q_scale=BASE + (6 << 30) + 8192, rows=4, cache_rows=4, ld_q=4 * 64, ld_kv=2 * 64, ld_cache=2 * 64,
             head_dim=64, hq=4, hk=2)
    d.update(kw)
    return ds.ds_qkseg(**d)


def call_qk(segs, eps=1e-6):
    arr = (ds.ds_qkseg * max(1, len(segs)))(*segs)
    return ds.lib().ds_qk_rows_l2(arr, len(segs), ct.c_float(eps), None)


def test_qk_validation():
    E = ds
    before = ds.ds_launch_count()
    assert call_qk([qkseg(head_dim=48, ld_q=4 * 48, ld_kv=96, ld_cache=96)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(head_dim=1024, ld_q=4096, ld_kv=2048, ld_cache=2048)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(hq=0, hk=0)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(hk=0, v=BASE + (2 << 30))]) == E.DS_ERR_INVALID_ARG   # v without k heads
    assert call_qk([qkseg(rows=-1)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(pos=None)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(inv_freq=None)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(q=None)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(k_cache=None)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(v_cache=None)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(ld_q=4 * 64 - 8)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(ld_cache=64)]) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(cache_rows=3)]) == E.DS_ERR_INVALID_ARG                # rows above cache rows, no slot
    assert call_qk([qkseg(q=BASE + 2)]) == E.DS_ERR_ALIGNMENT
    assert call_qk([qkseg(q_scale=BASE + (6 << 30) + 8192 + 4)]) == E.DS_ERR_ALIGNMENT
    assert call_qk([qkseg(pos=BASE + (6 << 30) + 2)]) == E.DS_ERR_ALIGNMENT
    assert call_qk([qkseg(q_out=BASE + 16)]) == E.DS_ERR_OVERLAP                 # partial overlap with q
    assert call_qk([qkseg(k_cache=BASE + (1 << 30), slot=BASE + (7 << 30))]) == E.DS_ERR_OVERLAP  # k in place with slots
    assert call_qk([qkseg(v_cache=BASE + (4 << 30))]) == E.DS_ERR_OVERLAP        # the two caches
    assert call_qk([qkseg()], eps=float("nan")) == E.DS_ERR_INVALID_ARG
    assert call_qk([qkseg(rows=0, q=None, k=None, pos=None)]) == E.DS_OK
    assert ds.ds_launch_count() == before


def test_qk_shifted_cache_alias_refused():
    """k_cache may be exactly k (row for row); a cache that starts one row
    into k overlaps it and is refused before anything runs."""
    assert call_qk([qkseg(k_cache=BASE + (1 << 30) + 128)]) == ds.DS_ERR_OVERLAP


# ------------------------------------------- scalar gain and row lengths --

def test_scalar_gain_and_row_norm_validation():
    E = ds
    before = ds.ds_launch_count()
    assert call_w("ds_wn_forward", [wseg(gain=None, gain_scalar=1)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_forward", [wseg(gain_scalar=2)]) == E.DS_ERR_INVALID_ARG
    arr = (ds.ds_wseg * 1)(wseg(rnorm=None))
    assert ds.lib().ds_row_norms(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
    arr = (ds.ds_wseg * 1)(wseg(rnorm=BASE + (5 << 30) + 2))
    assert ds.lib().ds_row_norms(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_ALIGNMENT
    arr = (ds.ds_wseg * 1)(wseg(rnorm=BASE + 64))                  # inside w
    assert ds.lib().ds_row_norms(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_OVERLAP
    arr = (ds.ds_wseg * 1)(wseg(rnorm=BASE + (5 << 30), radius=0.0))
    assert ds.lib().ds_gain_preserve(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
    assert ds.ds_launch_count() == before


def test_transposed_validation():
    E = ds
    before = ds.ds_launch_count()
    # stored [cols, ld] with ld >= rows: rows 8, cols 4 -> ld 8 is fine, ld 4 is not
    assert call_w("ds_wn_forward", [wseg(transposed=1, rows=8, cols=4, ld=4, ld_out=8)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_forward", [wseg(transposed=1, rows=8, cols=4, ld=8, ld_out=4)]) == E.DS_ERR_INVALID_ARG
    assert call_w("ds_wn_forward", [wseg(transposed=2)]) == E.DS_ERR_INVALID_ARG
    arr = (ds.ds_wseg * 1)(wseg(transposed=1, rnorm=BASE + (5 << 30)))
    assert ds.lib().ds_row_norms(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
    assert ds.ds_launch_count() == before


def test_grouped_transposed_validation():
    """ConvTranspose rows (transposed with tgroup G): cols a multiple of G,
    ld and ld_out >= rows * G, 1 <= G <= 256, and no tgroup without
    transposed; row lengths refuse them."""
    E = ds
    before = ds.ds_launch_count()
    # rows 4 of G = 2 columns each: stored [cols / 2, ld] with ld >= 8
    ok = dict(transposed=1, tgroup=2, rows=4, cols=8, ld=8, ld_out=8)
    bad = [dict(ok, tgroup=3),                       # 8 is not a multiple of 3
           dict(ok, ld=7), dict(ok, ld_out=7),      # < rows * G
           dict(ok, tgroup=257), dict(ok, tgroup=-1),
           dict(transposed=0, tgroup=2)]
    for kw in bad:
        assert call_w("ds_wn_forward", [wseg(**kw)]) == E.DS_ERR_INVALID_ARG, kw
        assert call_w("ds_wn_backward", [wseg(**kw)]) == E.DS_ERR_INVALID_ARG, kw
    arr = (ds.ds_wseg * 1)(wseg(tgroup=2, rnorm=BASE + (5 << 30)))
    assert ds.lib().ds_row_norms(arr, 1, ct.c_float(1e-6), None) == E.DS_ERR_INVALID_ARG
    assert ds.ds_launch_count() == before


def test_python_segments_map_shapes():
    """The binding's segment builders: a transposed weight gives rows = its
    stored columns; q/k segments count heads from the widths and refuse a
    width that is not whole heads.  (Host memory only: nothing is launched.)"""
    import torch

    w = torch.zeros(6, 10)                       # stored [in = 6, out = 10]
    c = ds.WSeg(w=w, transposed=True).to_c()
    assert (c.rows, c.cols, c.ld, c.transposed) == (10, 6, 10, 1)
    c = ds.WSeg(w=w).to_c()
    assert (c.rows, c.cols, c.transposed) == (6, 10, 0)
    # a ConvTranspose1d weight [in = 6, out = 5, k = 2] viewed as [6, 10]
    c = ds.WSeg(w=w, transposed=True, tgroup=2).to_c()
    assert (c.rows, c.cols, c.ld, c.transposed, c.tgroup) == (5, 12, 10, 1, 2)
    with pytest.raises(ValueError):
        ds.WSeg(w=w, transposed=True, tgroup=3).to_c()
    q = torch.zeros(3, 4 * 64, dtype=torch.bfloat16)
    k = torch.zeros(3, 2 * 64, dtype=torch.bfloat16)
    pos = torch.zeros(3, dtype=torch.int32)
    inv = torch.zeros(32)
    c = ds.QKSeg(head_dim=64, pos=pos, inv_freq=inv, q=q, q_out=q, k=k, k_cache=k).to_c()
    assert (c.rows, c.hq, c.hk, c.head_dim, c.ld_q, c.ld_kv, c.cache_rows) == (3, 4, 2, 64, 256, 128, 3)
    with pytest.raises(ValueError):
        ds.QKSeg(head_dim=64, pos=pos, inv_freq=inv, q=torch.zeros(3, 100, dtype=torch.bfloat16)).to_c()
