"""numpy front end of liboracle.so (ctypes).  Test infrastructure only.

Arrays are passed as 2-D numpy views (row stride = leading dimension); bf16
tensors travel as their uint16 bit patterns.  Outputs are dense [R, C].
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np

from . import build as _build

OR_DROP_SUM_ROUND = 0x01
OR_DROP_SLERP_A = 0x02
OR_DROP_SLERP_B = 0x04
OR_EPS_OUTSIDE = 0x08
OR_EPS_ZERO = 0x10
OR_BWD_PRINTED = 0x20
OR_DROP_GATED = 0x40
OR_DROP_SGATE = 0x80
OR_DROP_SUP = 0x100
OR_DROP_PRODUCT = 0x200
OR_DROP_ROT = 0x400
OR_DROP_QNORM = 0x800

_lib = None


def lib() -> ct.CDLL:
    global _lib
    if _lib is None:
        _lib = ct.CDLL(_build.build())
        i64, dbl, uns, vp, i32 = ct.c_int64, ct.c_double, ct.c_uint, ct.c_void_p, ct.c_int
        _lib.or_bf16_rne.argtypes = [dbl]
        _lib.or_bf16_rne.restype = ct.c_uint16
        _lib.or_bf16_value.argtypes = [ct.c_uint16]
        _lib.or_bf16_value.restype = dbl
        _lib.or_bf16_rne_array.argtypes = [vp, i64, vp]
        for name, n in (("or_sigmoid", 1), ("or_silu", 1)):
            getattr(_lib, name).argtypes = [dbl] * n
            getattr(_lib, name).restype = dbl
        _lib.or_gate_value.argtypes = [dbl, dbl, dbl, uns]
        _lib.or_gate_value.restype = dbl
        _lib.or_swiglu_value.argtypes = [dbl, dbl, dbl, dbl, uns]
        _lib.or_swiglu_value.restype = dbl
        _lib.or_bf16_rne_array.restype = None
        _lib.or_wn_forward.argtypes = [vp, i64, i64, i64, vp, dbl, dbl, uns, vp, i32]
        _lib.or_wn_backward.argtypes = [vp, i64, i64, i64, vp, i32, i64, vp, dbl, dbl, uns, vp, vp, i32]
        _lib.or_row_renorm.argtypes = [vp, i64, i64, i64, dbl, dbl, uns, vp, i32]
        _lib.or_grad_project.argtypes = [vp, i64, i64, i64, vp, i64, dbl, uns, vp, i32]
        _lib.or_renorm_momentum.argtypes = [vp, i64, i64, i64, vp, i64, dbl, dbl, uns, vp, vp, i32]
        _lib.or_grad_project_row.argtypes = [vp, vp, i64, dbl, uns, vp]
        _lib.or_grad_project_row.restype = None
        _lib.or_l2_rows.argtypes = [vp, vp, i64, i64, i64, dbl, uns, vp, vp, i32]
        _lib.or_l2_rows_backward.argtypes = [vp, vp, vp, i64, i64, i64, dbl, uns, vp, i32]
        _lib.or_gate_l2_rows.argtypes = [vp, vp, vp, i64, i64, i64, dbl, uns, vp, vp, i32]
        _lib.or_swiglu_l2_rows.argtypes = [vp, vp, vp, vp, i64, i64, i64, dbl, uns, vp, vp, i32]
        _lib.or_gate_l2_rows_interval.argtypes = [vp, vp, vp, i64, i64, i64, dbl, dbl, uns, vp, vp, i32]
        _lib.or_swiglu_l2_rows_interval.argtypes = [vp, vp, vp, vp, i64, i64, i64, dbl, dbl, uns, vp, vp, i32]
        _lib.or_row_norms.argtypes = [vp, i64, i64, i64, dbl, dbl, vp, i32]
        _lib.or_wn_backward_scalar_gain.argtypes = [vp, i64, i64, i64, vp, i32, i64, ct.c_float, dbl, dbl, uns, vp,
                                                    vp, vp, i32]
        _lib.or_qk_rows_l2.argtypes = [vp, i64, vp, i64, i64, i32, i32, i32, vp, vp, vp, dbl, uns, vp, vp, vp, vp,
                                       i32]
        _lib.or_qk_rows_l2_interval.argtypes = [vp, i64, vp, i64, i64, i32, i32, i32, vp, vp, vp, dbl, dbl, uns, vp,
                                                vp, vp, vp, i32]
        _lib.or_slerp_rows_backward.argtypes = [vp, vp, vp, vp, i64, i64, i64, dbl, uns, vp, vp, vp, i32]
        _lib.or_l2_row.argtypes = [vp, vp, i64, dbl, uns, vp, vp, vp]
        _lib.or_l2_row.restype = None
        _lib.or_slerp_row.argtypes = [vp, vp, vp, i64, dbl, uns, vp, vp, vp]
        _lib.or_slerp_row.restype = None
        _lib.or_l2_backward_row.argtypes = [vp, vp, vp, i64, dbl, uns, vp, vp]
        _lib.or_l2_backward_row.restype = None
        _lib.or_slerp_backward_row.argtypes = [vp, vp, vp, vp, i64, dbl, uns, vp, vp, vp, vp]
        _lib.or_slerp_backward_row.restype = None
        _lib.or_slerp_rows.argtypes = [vp, vp, vp, i64, i64, i64, dbl, uns, vp, vp, i32]
        _lib.or_wn_backward_row.argtypes = [vp, vp, i64, dbl, dbl, dbl, uns, vp, vp]
        _lib.or_wn_forward_row.argtypes = [vp, i64, dbl, dbl, dbl, uns, vp]
        _lib.or_l2_rows_interval.argtypes = [vp, vp, i64, i64, i64, dbl, dbl, uns, vp, vp, i32]
        _lib.or_slerp_rows_interval.argtypes = [vp, vp, vp, i64, i64, i64, dbl, dbl, uns, vp, vp, i32]
        for f in ("or_wn_forward", "or_wn_backward", "or_row_renorm", "or_l2_rows", "or_slerp_rows",
                  "or_l2_rows_interval", "or_slerp_rows_interval", "or_qk_rows_l2", "or_qk_rows_l2_interval",
                  "or_row_norms", "or_wn_backward_scalar_gain"):
            getattr(_lib, f).restype = i32
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _rows(a: np.ndarray, dtype) -> tuple[np.ndarray, int]:
    """Check a 2-D row-major view with unit column stride; return (a, ld)."""
    if a.dtype != dtype or a.ndim != 2:
        raise TypeError(f"expected 2-D {np.dtype(dtype)}, got {a.dtype} {a.shape}")
    if a.shape[0] == 0:
        return a, a.shape[1]
    if a.strides[1] != a.itemsize or a.strides[0] % a.itemsize:
        a = np.ascontiguousarray(a)
    return a, a.strides[0] // a.itemsize if a.shape[0] > 1 else a.shape[1]


def _p(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


def _check(rc: int, name: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments")


def bf16_rne(v: float) -> int:
    return int(lib().or_bf16_rne(float(v)))


def bf16_rne_array(a) -> np.ndarray:
    """Round every double of `a` straight to bf16 bits (same shape, uint16)."""
    src = np.ascontiguousarray(a, np.float64)
    dst = np.empty(src.shape, np.uint16)
    lib().or_bf16_rne_array(_p(src), src.size, _p(dst))
    return dst


def bf16_value(bits: int) -> float:
    return float(lib().or_bf16_value(int(bits) & 0xFFFF))


def sigmoid(z: float) -> float:
    """The oracle's sigmoid, 1/(1+exp(-z)) in double."""
    return lib().or_sigmoid(float(z))


def silu(x: float) -> float:
    """The oracle's silu, x/(1+exp(-x)) in double."""
    return lib().or_silu(float(x))


def gate_value(o: float, g: float, sg: float, flags: int = 0) -> float:
    """One element of the gated row: bf16(o sigmoid(g sg)) (OR_DROP_GATED: unrounded)."""
    return lib().or_gate_value(float(o), float(g), float(sg), flags)


def swiglu_value(g: float, u: float, sug: float, suu: float, flags: int = 0) -> float:
    """One element of the SwiGLU row: bf16(silu(bf16(g sug)) bf16(u suu))."""
    return lib().or_swiglu_value(float(g), float(u), float(sug), float(suu), flags)


def wn_forward(w, g=None, *, rho=1.0, eps=1e-6, flags=0, nthreads=1):
    """f64 W_eff [R, C] for fp32 rows w [R, C] (g fp32 [R] or None)."""
    w, ld = _rows(w, np.float32)
    R, C = w.shape
    out = np.empty((R, C), np.float64)
    g = None if g is None else np.ascontiguousarray(g, np.float32)
    _check(lib().or_wn_forward(_p(w), R, C, ld, _p(g), rho, eps, flags, _p(out), nthreads), "wn_forward")
    return out


def wn_backward(w, gy, g=None, *, rho=1.0, eps=1e-6, flags=0, nthreads=1):
    """f64 (grad_w [R, C], grad_g [R]); gy fp32 or bf16 bits (uint16)."""
    w, ld = _rows(w, np.float32)
    is_bf16 = gy.dtype == np.uint16
    gy, ldg = _rows(gy, np.uint16 if is_bf16 else np.float32)
    R, C = w.shape
    if gy.shape != (R, C):
        raise ValueError("gy shape")
    gw = np.empty((R, C), np.float64)
    gg = np.empty((R,), np.float64)
    g = None if g is None else np.ascontiguousarray(g, np.float32)
    _check(lib().or_wn_backward(_p(w), R, C, ld, _p(gy), int(is_bf16), ldg, _p(g), rho, eps, flags,
                                _p(gw), _p(gg), nthreads), "wn_backward")
    return gw, gg


def row_norms(w, *, eps=1e-6, div=1.0):
    """f64 [R]: sqrt(sum_j w[r,j]^2 + eps) / div (div = rho: the preserving gain)."""
    w, ld = _rows(w, np.float32)
    R, C = w.shape
    out = np.empty((R,), np.float64)
    _check(lib().or_row_norms(_p(w), R, C, ld, eps, div, _p(out), 1), "row_norms")
    return out


def wn_backward_scalar_gain(w, gy, g, *, rho=1.0, eps=1e-6, flags=0, nthreads=1):
    """f64 (grad_w [R, C], per-row gain gradients [R], their sum) for one
    scalar gain g shared by every row."""
    w, ld = _rows(w, np.float32)
    is_bf16 = gy.dtype == np.uint16
    gy, ldg = _rows(gy, np.uint16 if is_bf16 else np.float32)
    R, C = w.shape
    gw = np.empty((R, C), np.float64)
    gg = np.empty((R,), np.float64)
    tot = ct.c_double()
    _check(lib().or_wn_backward_scalar_gain(_p(w), R, C, ld, _p(gy), int(is_bf16), ldg, float(g), rho, eps, flags,
                                            _p(gw), _p(gg), ct.byref(tot), nthreads), "wn_backward_scalar_gain")
    return gw, gg, tot.value


def row_renorm(w, *, rho=1.0, eps=1e-6, flags=0, nthreads=1):
    w, ld = _rows(w, np.float32)
    R, C = w.shape
    out = np.empty((R, C), np.float64)
    _check(lib().or_row_renorm(_p(w), R, C, ld, rho, eps, flags, _p(out), nthreads), "row_renorm")
    return out


def l2_rows(x, r=None, *, eps=1e-6, flags=0, nthreads=1, exact=False):
    """bf16 bits y [R, C] (uint16); with exact=True also the f64 value before rounding."""
    x, ld = _rows(x, np.uint16)
    R, C = x.shape
    if r is not None:
        r, ldr = _rows(r, np.uint16)
        if r.shape != x.shape:
            raise ValueError("r shape")
        if ldr != ld:
            x, r = np.ascontiguousarray(x), np.ascontiguousarray(r)
            ld = C
    y = np.empty((R, C), np.uint16)
    ye = np.empty((R, C), np.float64) if exact else None
    _check(lib().or_l2_rows(_p(x), _p(r), R, C, ld, eps, flags, _p(y), _p(ye), nthreads), "l2_rows")
    return (y, ye) if exact else y


def slerp_rows(res, out, alpha, *, eps=1e-6, flags=0, nthreads=1, exact=False):
    res, ld = _rows(res, np.uint16)
    out, ldo = _rows(out, np.uint16)
    if out.shape != res.shape:
        raise ValueError("out shape")
    if ldo != ld:
        res, out = np.ascontiguousarray(res), np.ascontiguousarray(out)
        ld = res.shape[1]
    R, C = res.shape
    alpha = np.ascontiguousarray(alpha, np.float32)
    if alpha.shape != (C,):
        raise ValueError("alpha shape")
    h = np.empty((R, C), np.uint16)
    he = np.empty((R, C), np.float64) if exact else None
    _check(lib().or_slerp_rows(_p(res), _p(out), _p(alpha), R, C, ld, eps, flags, _p(h), _p(he), nthreads),
           "slerp_rows")
    return (h, he) if exact else h


def _fused_args(a, b, *vecs):
    a = np.ascontiguousarray(a, np.uint16)
    b = np.ascontiguousarray(b, np.uint16)
    R, C = a.shape
    if b.shape != (R, C):
        raise ValueError("shapes")
    vs = [np.ascontiguousarray(v, np.float32) for v in vecs]
    if any(v.shape != (C,) for v in vs):
        raise ValueError("scale vector shape")
    return a, b, vs, R, C


def gate_l2_rows(o, g, sg, *, eps=1e-6, flags=0, nthreads=1, exact=False):
    """bf16 bits y of bf16(l2(bf16(o * sigmoid(g * sg)))) (o, g bf16 bits, sg fp32 [C])."""
    o, g, (sg,), R, C = _fused_args(o, g, sg)
    y = np.empty((R, C), np.uint16)
    ye = np.empty((R, C), np.float64) if exact else None
    _check(lib().or_gate_l2_rows(_p(o), _p(g), _p(sg), R, C, C, eps, flags, _p(y), _p(ye), nthreads), "gate_l2")
    return (y, ye) if exact else y


def swiglu_l2_rows(g, u, sug, suu, *, eps=1e-6, flags=0, nthreads=1, exact=False):
    """bf16 bits y of bf16(l2(bf16(silu(bf16(g * sug)) * bf16(u * suu))))."""
    g, u, (sug, suu), R, C = _fused_args(g, u, sug, suu)
    y = np.empty((R, C), np.uint16)
    ye = np.empty((R, C), np.float64) if exact else None
    _check(lib().or_swiglu_l2_rows(_p(g), _p(u), _p(sug), _p(suu), R, C, C, eps, flags, _p(y), _p(ye), nthreads),
           "swiglu_l2")
    return (y, ye) if exact else y


def gate_l2_rows_interval(o, g, sg, *, eps=1e-6, delta=1e-5, flags=0, nthreads=1):
    o, g, (sg,), R, C = _fused_args(o, g, sg)
    lo = np.empty((R, C), np.uint16)
    hi = np.empty((R, C), np.uint16)
    _check(lib().or_gate_l2_rows_interval(_p(o), _p(g), _p(sg), R, C, C, eps, delta, flags, _p(lo), _p(hi),
                                          nthreads), "gate_l2_interval")
    return lo, hi


def swiglu_l2_rows_interval(g, u, sug, suu, *, eps=1e-6, delta=1e-5, flags=0, nthreads=1):
    g, u, (sug, suu), R, C = _fused_args(g, u, sug, suu)
    lo = np.empty((R, C), np.uint16)
    hi = np.empty((R, C), np.uint16)
    _check(lib().or_swiglu_l2_rows_interval(_p(g), _p(u), _p(sug), _p(suu), R, C, C, eps, delta, flags, _p(lo),
                                            _p(hi), nthreads), "swiglu_l2_interval")
    return lo, hi


def _qk_args(q, k, pos, inv, q_scale, head_dim):
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    if q.ndim != 2 or k.ndim != 2 or q.shape[0] != k.shape[0]:
        raise ValueError("q and k must be [R, heads * head_dim] with the same R")
    R = q.shape[0]
    if q.shape[1] % head_dim or k.shape[1] % head_dim:
        raise ValueError("widths must be whole heads")
    pos = np.ascontiguousarray(pos, np.int32)
    inv = np.ascontiguousarray(inv, np.float32)
    if pos.shape != (R,) or inv.shape != (head_dim // 2,):
        raise ValueError("pos [R], inv [head_dim / 2]")
    if q_scale is not None:
        q_scale = np.ascontiguousarray(q_scale, np.float32)
        if q_scale.shape != (q.shape[1],):
            raise ValueError("q_scale [hq * head_dim]")
    return q, k, pos, inv, q_scale, R, q.shape[1] // head_dim, k.shape[1] // head_dim


def qk_rows_l2(q, k, pos, inv, q_scale=None, *, head_dim, eps=1e-6, flags=0, nthreads=1, exact=False):
    """(q_out, k_out) bf16 bits of Dory's q and k rows: rotate-half RoPE at the
    fp32 angles fp32(pos * inv), per-head l2 with eps, q times q_scale
    (fp32 [hq * head_dim] or None).  q [R, hq*D], k [R, hk*D] bf16 bits."""
    q, k, pos, inv, sc, R, hq, hk = _qk_args(q, k, pos, inv, q_scale, head_dim)
    qo = np.empty((R, hq * head_dim), np.uint16)
    ko = np.empty((R, hk * head_dim), np.uint16)
    qe = np.empty(qo.shape, np.float64) if exact else None
    ke = np.empty(ko.shape, np.float64) if exact else None
    _check(lib().or_qk_rows_l2(_p(q), q.shape[1], _p(k), k.shape[1], R, head_dim, hq, hk, _p(pos), _p(inv), _p(sc),
                               eps, flags, _p(qo), _p(ko), _p(qe), _p(ke), nthreads), "qk_rows_l2")
    return (qo, ko, qe, ke) if exact else (qo, ko)


def qk_rows_l2_interval(q, k, pos, inv, q_scale=None, *, head_dim, eps=1e-6, delta=1e-5, flags=0, nthreads=1):
    """(q_lo, q_hi, k_lo, k_hi): the bf16 ends each output can reach."""
    q, k, pos, inv, sc, R, hq, hk = _qk_args(q, k, pos, inv, q_scale, head_dim)
    out = [np.empty((R, h * head_dim), np.uint16) for h in (hq, hq, hk, hk)]
    _check(lib().or_qk_rows_l2_interval(_p(q), q.shape[1], _p(k), k.shape[1], R, head_dim, hq, hk, _p(pos), _p(inv),
                                        _p(sc), eps, delta, flags, *[_p(o) for o in out], nthreads),
           "qk_rows_l2_interval")
    return tuple(out)


def l2_rows_backward(x, r, dy, *, eps=1e-6, flags=0, nthreads=1):
    """f64 dx [R, C] of l2_rows (x, r, dy: bf16 bits; r may be None).  With a
    residual the same values are the gradient of r."""
    x, ld = _rows(x, np.uint16)
    R, C = x.shape
    arrs = [x, np.ascontiguousarray(dy, np.uint16)] + ([] if r is None else [np.ascontiguousarray(r, np.uint16)])
    if any(a.shape != (R, C) for a in arrs):
        raise ValueError("shapes")
    x = np.ascontiguousarray(x)
    dy = arrs[1]
    r = None if r is None else arrs[2]
    dx = np.empty((R, C), np.float64)
    _check(lib().or_l2_rows_backward(_p(x), _p(r), _p(dy), R, C, C, eps, flags, _p(dx), nthreads),
           "l2_rows_backward")
    return dx


def slerp_rows_backward(res, out, alpha, dh, *, eps=1e-6, flags=0, nthreads=1, dalpha=True):
    """f64 (dres, dout, dalpha | None) of slerp_rows (bf16 bits in)."""
    res = np.ascontiguousarray(res, np.uint16)
    out = np.ascontiguousarray(out, np.uint16)
    dh = np.ascontiguousarray(dh, np.uint16)
    R, C = res.shape
    if out.shape != (R, C) or dh.shape != (R, C):
        raise ValueError("shapes")
    alpha = np.ascontiguousarray(alpha, np.float32)
    if alpha.shape != (C,):
        raise ValueError("alpha shape")
    dres = np.empty((R, C), np.float64)
    dout = np.empty((R, C), np.float64)
    da = np.empty((C,), np.float64) if dalpha else None
    _check(lib().or_slerp_rows_backward(_p(res), _p(out), _p(alpha), _p(dh), R, C, C, eps, flags, _p(dres),
                                        _p(dout), _p(da), nthreads), "slerp_rows_backward")
    return dres, dout, da


def l2_row64(x, r=None, *, eps=1e-6, flags=0):
    """One row with f64 inputs: the exact value before the output rounding."""
    x = np.ascontiguousarray(x, np.float64)
    r = None if r is None else np.ascontiguousarray(r, np.float64)
    s = np.empty_like(x)
    y = np.empty(x.shape, np.uint16)
    ye = np.empty_like(x)
    lib().or_l2_row(_p(x), _p(r), x.size, eps, flags, _p(s), _p(y), _p(ye))
    return ye


def slerp_row64(res, out, alpha, *, eps=1e-6, flags=0):
    res = np.ascontiguousarray(res, np.float64)
    out = np.ascontiguousarray(out, np.float64)
    alpha = np.ascontiguousarray(alpha, np.float64)
    tmp = np.empty(3 * res.size, np.float64)
    h = np.empty(res.shape, np.uint16)
    he = np.empty_like(res)
    lib().or_slerp_row(_p(res), _p(out), _p(alpha), res.size, eps, flags, _p(tmp), _p(h), _p(he))
    return he


def l2_backward_row64(x, r, dy, *, eps=1e-6, flags=0):
    x = np.ascontiguousarray(x, np.float64)
    r = None if r is None else np.ascontiguousarray(r, np.float64)
    dy = np.ascontiguousarray(dy, np.float64)
    s = np.empty_like(x)
    dx = np.empty_like(x)
    lib().or_l2_backward_row(_p(x), _p(r), _p(dy), x.size, eps, flags, _p(s), _p(dx))
    return dx


def slerp_backward_row64(res, out, alpha, dh, *, eps=1e-6, flags=0):
    res = np.ascontiguousarray(res, np.float64)
    out = np.ascontiguousarray(out, np.float64)
    alpha = np.ascontiguousarray(alpha, np.float64)
    dh = np.ascontiguousarray(dh, np.float64)
    tmp = np.empty(4 * res.size, np.float64)
    dres, dout, da = np.empty_like(res), np.empty_like(res), np.empty_like(res)
    lib().or_slerp_backward_row(_p(res), _p(out), _p(alpha), _p(dh), res.size, eps, flags, _p(tmp), _p(dres),
                                _p(dout), _p(da))
    return dres, dout, da


def l2_rows_interval(x, r=None, *, eps=1e-6, delta=1e-5, flags=0, nthreads=1):
    """(lo, hi) bf16 bits: the outputs any fp32 evaluation within relative
    `delta` per step can produce (TensorFold's range over the fp32 spread)."""
    x, ld = _rows(x, np.uint16)
    R, C = x.shape
    if r is not None:
        r, ldr = _rows(r, np.uint16)
        if ldr != ld:
            x, r = np.ascontiguousarray(x), np.ascontiguousarray(r)
            ld = C
    lo = np.empty((R, C), np.uint16)
    hi = np.empty((R, C), np.uint16)
    _check(lib().or_l2_rows_interval(_p(x), _p(r), R, C, ld, eps, delta, flags, _p(lo), _p(hi), nthreads),
           "l2_rows_interval")
    return lo, hi


def slerp_rows_interval(res, out, alpha, *, eps=1e-6, delta=1e-5, flags=0, nthreads=1):
    res, ld = _rows(res, np.uint16)
    out, ldo = _rows(out, np.uint16)
    if ldo != ld:
        res, out = np.ascontiguousarray(res), np.ascontiguousarray(out)
        ld = res.shape[1]
    R, C = res.shape
    alpha = np.ascontiguousarray(alpha, np.float32)
    lo = np.empty((R, C), np.uint16)
    hi = np.empty((R, C), np.uint16)
    _check(lib().or_slerp_rows_interval(_p(res), _p(out), _p(alpha), R, C, ld, eps, delta, flags, _p(lo), _p(hi),
                                        nthreads), "slerp_rows_interval")
    return lo, hi


def grad_project(w, G, *, eps=1e-6, flags=0, nthreads=1):
    """f64 G - w (w . G) / (S + eps) [R, C] for fp32 rows w and gradient G."""
    w, ld = _rows(w, np.float32)
    G, ldg = _rows(G, np.float32)
    R, C = w.shape
    if G.shape != (R, C):
        raise ValueError("G shape")
    out = np.empty((R, C), np.float64)
    _check(lib().or_grad_project(_p(w), R, C, ld, _p(G), ldg, eps, flags, _p(out), nthreads), "grad_project")
    return out


def renorm_momentum(w, m, *, rho=1.0, eps=1e-6, flags=0, nthreads=1):
    """f64 (w_out, m_out) [R, C]: m's component along the row removed and
    the row rescaled to its radius."""
    w, ld = _rows(w, np.float32)
    m, ldm = _rows(m, np.float32)
    R, C = w.shape
    if m.shape != (R, C):
        raise ValueError("m shape")
    wo = np.empty((R, C), np.float64)
    mo = np.empty((R, C), np.float64)
    _check(lib().or_renorm_momentum(_p(w), R, C, ld, _p(m), ldm, rho, eps, flags, _p(wo), _p(mo), nthreads),
           "renorm_momentum")
    return wo, mo


def grad_project_row64(w, G, *, eps=1e-6, flags=0):
    """One row with f64 inputs."""
    w = np.ascontiguousarray(w, np.float64)
    G = np.ascontiguousarray(G, np.float64)
    out = np.empty_like(w)
    lib().or_grad_project_row(_p(w), _p(G), w.size, eps, flags, _p(out))
    return out


def wn_forward_row64(w, g=1.0, *, rho=1.0, eps=1e-6, flags=0):
    """One row with f64 inputs (for finite differences)."""
    w = np.ascontiguousarray(w, np.float64)
    out = np.empty_like(w)
    lib().or_wn_forward_row(_p(w), w.size, float(g), rho, eps, flags, _p(out))
    return out


def wn_backward_row64(w, gy, g=1.0, *, rho=1.0, eps=1e-6, flags=0):
    w = np.ascontiguousarray(w, np.float64)
    gy = np.ascontiguousarray(gy, np.float64)
    gw = np.empty_like(w)
    gg = ct.c_double()
    lib().or_wn_backward_row(_p(w), _p(gy), w.size, float(g), rho, eps, flags, _p(gw), ct.byref(gg))
    return gw, gg.value


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "ct", "os", "np")]
