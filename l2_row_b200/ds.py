"""Thin ctypes binding of libds (include/ds.h): argument marshalling only.

Every step of the computation runs in the CUDA kernels of libds.so.  If the
library has not been built (``python -m l2_row_b200.build``) importing this
module raises: there is no CPU fallback.

The five calls keep their C names and take lists of segments:

    ds_wn_forward(segs, out_dtype, eps, stream=None)
    ds_wn_backward(segs, gy_dtype, eps, stream=None)
    ds_row_renorm(segs, eps, stream=None)
    ds_grad_project(segs, eps, stream=None)       (grad_w = the gradient, in place)
    ds_renorm_momentum(segs, eps, stream=None)    (grad_w = the momentum, in place)
    ds_l2_rows(segs, eps, stream=None)
    ds_slerp_rows(segs, eps, stream=None)
    ds_gate_l2_rows(segs, eps, stream=None)       (Dory's gated rows)
    ds_swiglu_l2_rows(segs, eps, stream=None)     (Dory's SwiGLU rows)
    ds_l2_rows_backward(segs, eps, stream=None)
    ds_slerp_rows_backward(segs, eps, dalpha=None, workspace=None, stream=None)

A segment is a ``WSeg`` / ``ASeg`` of CUDA tensors (2-D, unit column stride,
row stride = leading dimension) or a raw ``ds_wseg`` / ``ds_aseg`` structure.
``stream`` defaults to torch's current CUDA stream.  A failing call raises
``DSError`` carrying the status code and the library's message.
"""
from __future__ import annotations

import ctypes as ct
import os
from dataclasses import dataclass
from typing import Any, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libds.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libds.so is not built ({LIB_PATH}); run `python -m l2_row_b200.build`")

_lib = ct.CDLL(LIB_PATH)

DS_OK, DS_ERR_INVALID_ARG, DS_ERR_ALIGNMENT, DS_ERR_UNSUPPORTED_DTYPE = 0, 1, 2, 3
DS_ERR_TOO_MANY_SEGMENTS, DS_ERR_CUDA, DS_ERR_DEVICE_TIMEOUT, DS_ERR_OVERLAP = 4, 5, 6, 7
DS_F32, DS_BF16 = 0, 1
DS_OP_WN_FORWARD, DS_OP_WN_BACKWARD, DS_OP_ROW_RENORM, DS_OP_L2_ROWS, DS_OP_SLERP_ROWS = range(5)
DS_OP_GRAD_PROJECT, DS_OP_RENORM_MOMENTUM = 5, 6
DS_OP_L2_ROWS_BACKWARD, DS_OP_SLERP_ROWS_BACKWARD = 7, 8
DS_OP_GATE_L2_ROWS, DS_OP_SWIGLU_L2_ROWS = 9, 10
DS_PATH_AUTO, DS_PATH_WARP, DS_PATH_CTA, DS_PATH_CLUSTER, DS_PATH_TWO_PASS = range(5)
DS_MAX_SEGMENTS = 65536
PATH_NAMES = {DS_PATH_WARP: "warp", DS_PATH_CTA: "cta", DS_PATH_CLUSTER: "cluster", DS_PATH_TWO_PASS: "two_pass"}


class ds_wseg(ct.Structure):
    _fields_ = [("w", ct.c_void_p), ("gain", ct.c_void_p), ("w_eff", ct.c_void_p), ("gy", ct.c_void_p),
                ("grad_w", ct.c_void_p), ("grad_g", ct.c_void_p), ("rows", ct.c_int64), ("cols", ct.c_int64),
                ("ld", ct.c_int64), ("ld_out", ct.c_int64), ("radius", ct.c_float), ("gain_scalar", ct.c_int32),
                ("rnorm", ct.c_void_p), ("transposed", ct.c_int32), ("tgroup", ct.c_int32)]


class ds_aseg(ct.Structure):
    _fields_ = [("x", ct.c_void_p), ("r", ct.c_void_p), ("y", ct.c_void_p), ("alpha", ct.c_void_p),
                ("rows", ct.c_int64), ("cols", ct.c_int64), ("ld", ct.c_int64)]


class ds_fseg(ct.Structure):
    _fields_ = [("a", ct.c_void_p), ("b", ct.c_void_p), ("y", ct.c_void_p), ("sa", ct.c_void_p),
                ("sb", ct.c_void_p), ("rows", ct.c_int64), ("cols", ct.c_int64), ("ld", ct.c_int64)]


class ds_agseg(ct.Structure):
    _fields_ = [("x", ct.c_void_p), ("r", ct.c_void_p), ("dy", ct.c_void_p), ("dx", ct.c_void_p),
                ("dr", ct.c_void_p), ("alpha", ct.c_void_p), ("rows", ct.c_int64), ("cols", ct.c_int64),
                ("ld", ct.c_int64), ("ld_d", ct.c_int64)]


class ds_qkseg(ct.Structure):
    _fields_ = [("q", ct.c_void_p), ("k", ct.c_void_p), ("v", ct.c_void_p), ("q_out", ct.c_void_p),
                ("k_cache", ct.c_void_p), ("v_cache", ct.c_void_p), ("pos", ct.c_void_p), ("slot", ct.c_void_p),
                ("inv_freq", ct.c_void_p), ("q_scale", ct.c_void_p), ("rows", ct.c_int64),
                ("cache_rows", ct.c_int64), ("ld_q", ct.c_int64), ("ld_kv", ct.c_int64), ("ld_cache", ct.c_int64),
                ("head_dim", ct.c_int32), ("hq", ct.c_int32), ("hk", ct.c_int32)]


_st = ct.c_int
_lib.ds_wn_forward.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_wn_backward.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_row_renorm.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_grad_project.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_renorm_momentum.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_l2_rows.argtypes = [ct.POINTER(ds_aseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_slerp_rows.argtypes = [ct.POINTER(ds_aseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_l2_rows_backward.argtypes = [ct.POINTER(ds_agseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_gate_l2_rows.argtypes = [ct.POINTER(ds_fseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_swiglu_l2_rows.argtypes = [ct.POINTER(ds_fseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_qk_rows_l2.argtypes = [ct.POINTER(ds_qkseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_row_norms.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_gain_preserve.argtypes = [ct.POINTER(ds_wseg), ct.c_int, ct.c_float, ct.c_void_p]
_lib.ds_slerp_rows_backward.argtypes = [ct.POINTER(ds_agseg), ct.c_int, ct.c_float, ct.c_void_p, ct.c_void_p,
                                        ct.c_uint64, ct.c_void_p]
_lib.ds_slerp_rows_backward_noalloc.argtypes = [ct.POINTER(ds_agseg), ct.c_int, ct.c_float, ct.c_void_p,
                                                ct.c_void_p]
_lib.ds_slerp_rows_backward_noalloc.restype = ct.c_int
_lib.ds_slerp_rows_backward_workspace.argtypes = [ct.c_int64]
_lib.ds_slerp_rows_backward_workspace.restype = ct.c_uint64
for _f in ("ds_wn_forward", "ds_wn_backward", "ds_row_renorm", "ds_grad_project", "ds_renorm_momentum",
           "ds_l2_rows", "ds_slerp_rows", "ds_l2_rows_backward", "ds_slerp_rows_backward",
           "ds_gate_l2_rows", "ds_swiglu_l2_rows", "ds_qk_rows_l2", "ds_row_norms", "ds_gain_preserve",
           "ds_get_device_status", "ds_row_class", "ds_debug_force_path", "ds_debug_set_wait_limit_ns",
           "ds_debug_wait_timeout_selftest", "ds_debug_division_check"):
    getattr(_lib, _f).restype = _st
_lib.ds_status_string.argtypes = [ct.c_int]
_lib.ds_status_string.restype = ct.c_char_p
_lib.ds_last_error.argtypes = []
_lib.ds_last_error.restype = ct.c_char_p
_lib.ds_get_device_status.argtypes = [ct.c_void_p]
_lib.ds_launch_count.argtypes = []
_lib.ds_launch_count.restype = ct.c_uint64
_lib.ds_version.argtypes = []
_lib.ds_version.restype = ct.c_int
_lib.ds_row_class.argtypes = [ct.c_int, ct.c_int64, ct.POINTER(ct.c_int), ct.POINTER(ct.c_int),
                              ct.POINTER(ct.c_int)]
_lib.ds_debug_force_path.argtypes = [ct.c_int]
_lib.ds_debug_set_wait_limit_ns.argtypes = [ct.c_uint64]
_lib.ds_debug_wait_timeout_selftest.argtypes = [ct.c_uint64, ct.c_void_p]
_lib.ds_debug_division_check.argtypes = [ct.c_void_p, ct.c_void_p]

#: every symbol include/ds.h declares
EXPORTS = ("ds_wn_forward", "ds_wn_backward", "ds_row_renorm", "ds_grad_project", "ds_renorm_momentum",
           "ds_l2_rows", "ds_slerp_rows", "ds_l2_rows_backward", "ds_slerp_rows_backward",
           "ds_gate_l2_rows", "ds_swiglu_l2_rows", "ds_qk_rows_l2", "ds_row_norms", "ds_gain_preserve",
           "ds_slerp_rows_backward_workspace", "ds_slerp_rows_backward_noalloc", "ds_status_string", "ds_last_error", "ds_get_device_status", "ds_launch_count", "ds_version",
           "ds_row_class", "ds_debug_force_path", "ds_debug_set_wait_limit_ns", "ds_debug_wait_timeout_selftest",
           "ds_debug_division_check")


def lib() -> ct.CDLL:
    """The loaded libds.so (for direct C-ABI calls)."""
    return _lib


class DSError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ds_status_string(status).decode()
        detail = _lib.ds_last_error().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail else ""))


def _check(status: int, where: str) -> None:
    if status != DS_OK:
        raise DSError(status, where)


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch

        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(dt) -> int:
    if isinstance(dt, int):
        return dt
    s = str(dt).replace("torch.", "")
    if s in ("bf16", "bfloat16"):
        return DS_BF16
    if s in ("f32", "float32", "float"):
        return DS_F32
    raise ValueError(f"unsupported dtype {dt!r}")


# ------------------------------------------------------------ tensor views --

def _mat(t, name: str, rows: int, cols: int) -> tuple[int, int]:
    """(data_ptr, leading dimension) of a 2-D row-major view; (0, cols) for None."""
    if t is None:
        return 0, cols
    if t.dim() != 2 or tuple(t.shape) != (rows, cols):
        raise ValueError(f"{name}: expected shape ({rows}, {cols}), got {tuple(t.shape)}")
    if rows == 0:
        return t.data_ptr(), cols
    if t.stride(1) != 1 and cols > 1:
        raise ValueError(f"{name}: columns must be contiguous")
    return t.data_ptr(), (t.stride(0) if rows > 1 else max(t.stride(0), cols))


def _vec(t) -> int:
    if t is None:
        return 0
    if t.dim() != 1 or (t.numel() > 1 and t.stride(0) != 1):
        raise ValueError("per-row vectors must be contiguous 1-D tensors")
    return t.data_ptr()


@dataclass
class WSeg:
    """One weight matrix.  w: fp32 [R, C]; gain: fp32 [R] or None; w_eff:
    forward output [R, C]; gy, grad_w, grad_g: backward input/outputs.
    For ds_grad_project grad_w is the gradient and for ds_renorm_momentum
    the momentum buffer (fp32 [R, C], w's leading dimension, in place).
    gain_scalar: gain is fp32 [1] shared by every row and grad_g fp32 [R + 1]
    (per-row parts, then their sum).  rnorm: fp32 [R] output of
    ds_row_norms / ds_gain_preserve.  transposed: the unit rows are the
    columns of w (GPT-2 Conv1D, stored [in, out] = [C, R]); w, w_eff, gy and
    grad_w are then given in that stored layout.  tgroup (with transposed):
    G consecutive stored columns per unit row, for a ConvTranspose weight
    [in, out, k...] viewed as [in, out * G] (G = the kernel's volume): unit
    rows R = out, row length C = in * G."""

    w: Any
    gain: Any = None
    w_eff: Any = None
    gy: Any = None
    grad_w: Any = None
    grad_g: Any = None
    radius: float = 1.0
    gain_scalar: bool = False
    rnorm: Any = None
    transposed: bool = False
    tgroup: int = 1

    def to_c(self) -> ds_wseg:
        SR, SC = (int(self.w.shape[0]), int(self.w.shape[1]))   # the stored shape
        G = int(self.tgroup) if self.transposed else 1
        if G < 1 or SC % G:
            raise ValueError("tgroup must be >= 1 and divide the stored columns")
        R, C = (SC // G, SR * G) if self.transposed else (SR, SC)
        w, ld = _mat(self.w, "w", SR, SC)
        weff, ld_out = _mat(self.w_eff, "w_eff", SR, SC)
        gy, ld_gy = _mat(self.gy, "gy", SR, SC)
        gw, ld_gw = _mat(self.grad_w, "grad_w", SR, SC)
        if self.w_eff is not None and self.gy is not None and ld_out != ld_gy:
            raise ValueError("w_eff and gy must share a leading dimension")
        if self.grad_w is not None and ld_gw != ld:
            raise ValueError("grad_w must share w's leading dimension")
        return ds_wseg(w, _vec(self.gain), weff, gy, gw, _vec(self.grad_g), R, C, ld,
                       ld_out if self.w_eff is not None else ld_gy, float(self.radius), int(bool(self.gain_scalar)),
                       _vec(self.rnorm), int(bool(self.transposed)), G if self.transposed else 0)


@dataclass
class ASeg:
    """One activation matrix: x (slerp: res), r (slerp: out; l2: residual or
    None), y output, alpha fp32 [C] (slerp only).  bf16 [R, C], shared ld."""

    x: Any
    y: Any
    r: Any = None
    alpha: Any = None

    def to_c(self) -> ds_aseg:
        R, C = (int(self.x.shape[0]), int(self.x.shape[1]))
        x, ld = _mat(self.x, "x", R, C)
        y, ldy = _mat(self.y, "y", R, C)
        r, ldr = _mat(self.r, "r", R, C)
        if ldy != ld or (self.r is not None and ldr != ld):
            raise ValueError("x, r and y must share a leading dimension")
        return ds_aseg(x, r, y, _vec(self.alpha), R, C, ld)


@dataclass
class FSeg:
    """One activation matrix for Dory's rows: a, b, y bf16 [R, C] with a
    shared ld; sa (and for SwiGLU sb) fp32 [C].  Gate: a = o, b = g, sa = sg;
    SwiGLU: a = g, b = u, sa = sug, sb = suu."""

    a: Any
    b: Any
    y: Any
    sa: Any
    sb: Any = None

    def to_c(self) -> ds_fseg:
        R, C = (int(self.a.shape[0]), int(self.a.shape[1]))
        a, ld = _mat(self.a, "a", R, C)
        b, ldb = _mat(self.b, "b", R, C)
        y, ldy = _mat(self.y, "y", R, C)
        if ldb != ld or ldy != ld:
            raise ValueError("a, b and y must share a leading dimension")
        return ds_fseg(a, b, y, _vec(self.sa), _vec(self.sb), R, C, ld)


@dataclass
class QKSeg:
    """Dory's attention rows for ds_qk_rows_l2.  q [R, hq*D], k and v
    [R, hk*D] bf16; q_out [R, hq*D]; k_cache, v_cache [cache_rows, hk*D]
    (row slot[t], or t without slot, receives row t); pos, slot int32 [R];
    inv_freq fp32 [D/2]; q_scale fp32 [hq*D] or None.  Any of q/q_out or
    k/k_cache (v/v_cache) may be None when hq (hk) is 0."""

    head_dim: int
    pos: Any
    inv_freq: Any
    q: Any = None
    q_out: Any = None
    k: Any = None
    k_cache: Any = None
    v: Any = None
    v_cache: Any = None
    slot: Any = None
    q_scale: Any = None

    def to_c(self) -> ds_qkseg:
        D = int(self.head_dim)
        R = int(self.pos.shape[0])
        if self.q is not None:
            if self.q.shape[1] % D:
                raise ValueError("q: width is not a whole number of heads")
            hq = int(self.q.shape[1]) // D
        else:
            hq = 0
        if self.k is not None:
            if self.k.shape[1] % D:
                raise ValueError("k: width is not a whole number of heads")
            hk = int(self.k.shape[1]) // D
        else:
            hk = 0
        q, ld_q = _mat(self.q, "q", R, hq * D)
        qo, ld_qo = _mat(self.q_out, "q_out", R, hq * D)
        k, ld_kv = _mat(self.k, "k", R, hk * D)
        v, ld_v = _mat(self.v, "v", R, hk * D)
        C = 0 if self.k_cache is None else int(self.k_cache.shape[0])
        kc, ld_c = _mat(self.k_cache, "k_cache", C, hk * D)
        vc, ld_vc = _mat(self.v_cache, "v_cache", C, hk * D)
        if hq and ld_qo != ld_q:
            raise ValueError("q and q_out must share a leading dimension")
        if self.v is not None and ld_v != ld_kv:
            raise ValueError("k and v must share a leading dimension")
        if self.v_cache is not None and ld_vc != ld_c:
            raise ValueError("k_cache and v_cache must share a leading dimension")
        return ds_qkseg(q, k, v, qo, kc, vc, _vec(self.pos), _vec(self.slot), _vec(self.inv_freq),
                        _vec(self.q_scale), R, C, ld_q, ld_kv, ld_c, D, hq, hk)


@dataclass
class AGSeg:
    """One activation matrix for the backward calls: x (slerp: res), r (l2:
    residual or None; slerp: out), dy the upstream gradient (bf16 [R, C],
    shared ld), dx (and for slerp dr) fp32 [R, C] outputs with a shared ld,
    alpha fp32 [C] (slerp)."""

    x: Any
    dy: Any
    dx: Any
    r: Any = None
    dr: Any = None
    alpha: Any = None

    def to_c(self) -> ds_agseg:
        R, C = (int(self.x.shape[0]), int(self.x.shape[1]))
        x, ld = _mat(self.x, "x", R, C)
        dy, ldy = _mat(self.dy, "dy", R, C)
        r, ldr = _mat(self.r, "r", R, C)
        dx, ldd = _mat(self.dx, "dx", R, C)
        dr, lddr = _mat(self.dr, "dr", R, C)
        if ldy != ld or (self.r is not None and ldr != ld):
            raise ValueError("x, r and dy must share a leading dimension")
        if self.dr is not None and lddr != ldd:
            raise ValueError("dx and dr must share a leading dimension")
        return ds_agseg(x, r, dy, dx, dr, _vec(self.alpha), R, C, ld, ldd)


def _table(segs, cls):
    items = [s if isinstance(s, cls) else s.to_c() for s in segs]
    arr = (cls * max(1, len(items)))(*items)
    return arr, len(items)


def ds_wn_forward(segs: Sequence, out_dtype="bf16", eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_wn_forward(arr, n, _dtype_code(out_dtype), eps, _stream_ptr(stream)), "ds_wn_forward")


def ds_wn_backward(segs: Sequence, gy_dtype="bf16", eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_wn_backward(arr, n, _dtype_code(gy_dtype), eps, _stream_ptr(stream)), "ds_wn_backward")


def ds_row_renorm(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_row_renorm(arr, n, eps, _stream_ptr(stream)), "ds_row_renorm")


def ds_grad_project(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_grad_project(arr, n, eps, _stream_ptr(stream)), "ds_grad_project")


def ds_renorm_momentum(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_renorm_momentum(arr, n, eps, _stream_ptr(stream)), "ds_renorm_momentum")


def ds_l2_rows(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_aseg)
    _check(_lib.ds_l2_rows(arr, n, eps, _stream_ptr(stream)), "ds_l2_rows")


def ds_slerp_rows(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_aseg)
    _check(_lib.ds_slerp_rows(arr, n, eps, _stream_ptr(stream)), "ds_slerp_rows")


def ds_gate_l2_rows(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_fseg)
    _check(_lib.ds_gate_l2_rows(arr, n, eps, _stream_ptr(stream)), "ds_gate_l2_rows")


def ds_swiglu_l2_rows(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_fseg)
    _check(_lib.ds_swiglu_l2_rows(arr, n, eps, _stream_ptr(stream)), "ds_swiglu_l2_rows")


def ds_row_norms(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_row_norms(arr, n, eps, _stream_ptr(stream)), "ds_row_norms")


def ds_gain_preserve(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_wseg)
    _check(_lib.ds_gain_preserve(arr, n, eps, _stream_ptr(stream)), "ds_gain_preserve")


def ds_qk_rows_l2(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_qkseg)
    _check(_lib.ds_qk_rows_l2(arr, n, eps, _stream_ptr(stream)), "ds_qk_rows_l2")


def ds_l2_rows_backward(segs: Sequence, eps: float = 1e-6, stream=None) -> None:
    arr, n = _table(segs, ds_agseg)
    _check(_lib.ds_l2_rows_backward(arr, n, eps, _stream_ptr(stream)), "ds_l2_rows_backward")


def ds_slerp_rows_backward_workspace(cols: int) -> int:
    """Workspace bytes ds_slerp_rows_backward needs for dalpha over `cols` columns."""
    return int(_lib.ds_slerp_rows_backward_workspace(cols))


def ds_slerp_rows_backward(segs: Sequence, eps: float = 1e-6, dalpha=None, workspace=None, stream=None) -> None:
    """dalpha: fp32 [cols] CUDA tensor or None.  workspace: a CUDA tensor of at
    least ds_slerp_rows_backward_workspace(cols) bytes (256-byte aligned), or
    None to have one allocated here for this call."""
    arr, n = _table(segs, ds_agseg)
    ws_ptr, ws_bytes = 0, 0
    if dalpha is not None:
        cols = int(arr[0].cols) if n else 0
        need = ds_slerp_rows_backward_workspace(cols) if cols else 0
        if workspace is None and need:
            import torch

            workspace = torch.empty(need, dtype=torch.uint8, device=dalpha.device)
        if workspace is not None:
            ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    _check(_lib.ds_slerp_rows_backward(arr, n, eps, _vec(dalpha), ws_ptr, ws_bytes, _stream_ptr(stream)),
           "ds_slerp_rows_backward")


def ds_slerp_rows_backward_noalloc(segs: Sequence, eps: float = 1e-6, dalpha=None, stream=None) -> None:
    """ds_slerp_rows_backward for callers that cannot allocate device memory
    where they run the backward (their device memory all belongs to a pool
    of their own, or they must avoid the implicit synchronisation of
    cudaMalloc / cudaFree): dalpha's partial sums go to the library's
    built-in 64 MB scratch instead of a workspace.  Rows needing more than
    that are refused; calls must not overlap on the GPU."""
    arr, n = _table(segs, ds_agseg)
    _check(_lib.ds_slerp_rows_backward_noalloc(arr, n, eps, _vec(dalpha), _stream_ptr(stream)),
           "ds_slerp_rows_backward_noalloc")


def ds_get_device_status(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error word."""
    return int(_lib.ds_get_device_status(_stream_ptr(stream)))


def ds_launch_count() -> int:
    return int(_lib.ds_launch_count())


def ds_version() -> int:
    return int(_lib.ds_version())


def ds_status_string(status: int) -> str:
    return _lib.ds_status_string(status).decode()


def ds_last_error() -> str:
    return _lib.ds_last_error().decode()


def ds_row_class(op: int, cols: int) -> tuple[int, int, int]:
    """(path, threads per row, CTAs per row) the library picks for this row length."""
    p, g, c = ct.c_int(), ct.c_int(), ct.c_int()
    _check(_lib.ds_row_class(op, cols, ct.byref(p), ct.byref(g), ct.byref(c)), "ds_row_class")
    return p.value, g.value, c.value


def ds_debug_force_path(path: int) -> None:
    _check(_lib.ds_debug_force_path(path), "ds_debug_force_path")


def ds_debug_set_wait_limit_ns(limit_ns: int) -> None:
    _check(_lib.ds_debug_set_wait_limit_ns(limit_ns), "ds_debug_set_wait_limit_ns")


def ds_debug_wait_timeout_selftest(limit_ns: int, stream=None) -> None:
    _check(_lib.ds_debug_wait_timeout_selftest(limit_ns, _stream_ptr(stream)), "ds_debug_wait_timeout_selftest")


def ds_debug_division_check(stream=None) -> tuple[int, int, int, int]:
    """(reciprocal mismatches, quotient mismatches, reciprocal inputs checked,
    quotient inputs checked) of the Dory rows' fast division over every fp32
    input; synchronises the stream."""
    import torch

    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    _check(_lib.ds_debug_division_check(counts.data_ptr(), _stream_ptr(stream)), "ds_debug_division_check")
    torch.cuda.synchronize()
    return tuple(int(v) for v in counts.tolist())


class force_path:
    """Context manager: run the enclosed calls on one path (tests)."""

    def __init__(self, path: int):
        self.path = path

    def __enter__(self):
        ds_debug_force_path(self.path)
        return self

    def __exit__(self, *exc):
        ds_debug_force_path(DS_PATH_AUTO)
        return False
