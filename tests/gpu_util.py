"""GPU-side helpers for the parity tests: move seeded host inputs to the
device, run the five calls through the C ABI (l2_row_b200.ds), and compare
the results with the oracle by the rules in tests/checks.py."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests.checks import (SPREAD, bf16_interval_violations, bf16_key, bf16_ulp_violations, rel_violations)

DEV = "cuda"
CANARY_F32 = np.float32(-7.0e33)
CANARY_BF16 = 0x7BAD


# --------------------------------------------------------------- transfers --

def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16))
    return t.to(DEV).view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def padded(rows: int, cols: int, ld: int, dtype, canary) -> tuple[torch.Tensor, torch.Tensor]:
    """A [rows, cols] view with leading dimension ld inside a buffer that has
    one guard row before and after, every unused element set to `canary`.
    Returns (view, whole buffer)."""
    if dtype == torch.bfloat16:
        buf = torch.full(((rows + 2) * ld,), canary, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    else:
        buf = torch.full(((rows + 2) * ld,), float(canary), dtype=dtype, device=DEV)
    view = buf[ld:ld + rows * ld].view(rows, ld)[:, :cols] if rows else buf[:0].view(0, cols)
    return view, buf


def guards_intact(buf: torch.Tensor, rows: int, cols: int, ld: int, canary) -> bool:
    """Everything outside the [rows, cols] window still holds the canary."""
    if buf.dtype == torch.bfloat16:
        h = buf.view(torch.int16).cpu().numpy().view(np.uint16)
    else:
        h = buf.cpu().numpy()
    mask = np.ones(h.shape, bool)
    for r in range(rows):
        mask[(r + 1) * ld:(r + 1) * ld + cols] = False
    return bool(np.all(h[mask] == canary))


def copy_into(view: torch.Tensor, src: torch.Tensor) -> None:
    view.copy_(src)


# ---------------------------------------------------------------- running --

def run_forward(segs, out_dtype: str, eps: float, stream=None):
    """segs: list of WeightSeg (host).  Returns list of output tensors."""
    outs, cs = [], []
    for s in segs:
        w = dev_f32(s.w)
        g = dev_f32(s.g) if s.g is not None else None
        o = torch.empty(s.w.shape, dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32, device=DEV)
        cs.append(ds.WSeg(w=w, gain=g, w_eff=o, radius=s.radius))
        outs.append(o)
    ds.ds_wn_forward(cs, out_dtype, eps, stream)
    torch.cuda.synchronize()
    return outs


def run_backward(segs, gy_dtype: str, eps: float):
    res, cs = [], []
    for s in segs:
        w = dev_f32(s.w)
        g = dev_f32(s.g) if s.g is not None else None
        gy = dev_bf16(s.gy) if gy_dtype == "bf16" else dev_f32(s.gy)
        gw = torch.empty(s.w.shape, dtype=torch.float32, device=DEV)
        gg = torch.empty(s.w.shape[0], dtype=torch.float32, device=DEV) if g is not None else None
        cs.append(ds.WSeg(w=w, gain=g, gy=gy, grad_w=gw, grad_g=gg, radius=s.radius))
        res.append((gw, gg))
    ds.ds_wn_backward(cs, gy_dtype, eps)
    torch.cuda.synchronize()
    return res


def run_renorm(segs, eps: float):
    ws, cs = [], []
    for s in segs:
        w = dev_f32(s.w)
        cs.append(ds.WSeg(w=w, radius=s.radius))
        ws.append(w)
    ds.ds_row_renorm(cs, eps)
    torch.cuda.synchronize()
    return ws


def run_project(segs, eps: float):
    """ds_grad_project with seg.gy (fp32) as the gradient; returns the updated G tensors."""
    gs, cs = [], []
    for s in segs:
        G = dev_f32(s.gy)
        cs.append(ds.WSeg(w=dev_f32(s.w), grad_w=G))
        gs.append(G)
    ds.ds_grad_project(cs, eps)
    torch.cuda.synchronize()
    return gs


def run_momentum(segs, eps: float):
    """ds_renorm_momentum with seg.gy (fp32) as the momentum; returns (w, m) tensors."""
    res, cs = [], []
    for s in segs:
        w, m = dev_f32(s.w), dev_f32(s.gy)
        cs.append(ds.WSeg(w=w, grad_w=m, radius=s.radius))
        res.append((w, m))
    ds.ds_renorm_momentum(cs, eps)
    torch.cuda.synchronize()
    return res


def run_l2(acts, eps: float, residual: bool = True):
    ys, cs = [], []
    for a in acts:
        x = dev_bf16(a.x)
        r = dev_bf16(a.r) if (residual and a.r is not None) else None
        y = torch.empty_like(x)
        cs.append(ds.ASeg(x=x, r=r, y=y))
        ys.append(y)
    ds.ds_l2_rows(cs, eps)
    torch.cuda.synchronize()
    return ys


def run_slerp(acts, eps: float):
    hs, cs = [], []
    for a in acts:
        x, o = dev_bf16(a.x), dev_bf16(a.r)
        h = torch.empty_like(x)
        cs.append(ds.ASeg(x=x, r=o, y=h, alpha=dev_f32(a.alpha)))
        hs.append(h)
    ds.ds_slerp_rows(cs, eps)
    torch.cuda.synchronize()
    return hs


# ------------------------------------------------------------ comparisons --

def assert_bf16_rows(got_bits, ref_bits, lo=None, hi=None, what="", ambiguous=None) -> int:
    """Two separate rules; returns the number of outputs more than 1 ulp from
    the oracle's point value.

    * 1 ulp: every output is within 1 bf16 ulp of the oracle's bits, except
      where `ambiguous` (broadcastable mask) marks an element at which an
      intermediate rounding point of the definition lies within the fp32
      spread of a bf16 halfway point, so that either rounding of it is a
      value "rounded at the stated point".  Without a mask the count must
      be 0.
    * interval: where lo / hi are given, every output lies inside the
      oracle's interval (the range over the fp32 spread), so an excused
      output is still one of the legitimate fp32 outcomes."""
    far = bf16_ulp_violations(got_bits, ref_bits)
    n_far = int(far.sum())
    if lo is not None:
        outside = bf16_interval_violations(got_bits, lo, hi)
        assert not outside.any(), f"{what}: {int(outside.sum())} outputs outside the fp32-spread interval " \
                                  f"(first at {np.argwhere(outside)[0].tolist()})"
    bad = far if ambiguous is None else far & ~np.broadcast_to(ambiguous, far.shape)
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs beyond 1 bf16 ulp at elements with no ambiguous " \
                          f"rounding point (first at {np.argwhere(bad)[0].tolist()})"
    return n_far


def interval_admits_beyond_ulp(ref_bits, lo, hi) -> np.ndarray:
    """Elements at which the oracle's interval itself admits an output more
    than 1 ulp from its point value.  The interval widens each fp32 step by
    a relative 1e-5, about 400 times less than half a bf16 ulp, so this only
    happens where an intermediate rounding point of the definition is
    halfway-ambiguous (both of its roundings lie inside)."""
    k, kl, kh = bf16_key(ref_bits), bf16_key(lo), bf16_key(hi)
    return (k - kl > 1) | (kh - k > 1)


def slerp_ambiguous(x_bits, o_bits, eps: float, delta: float = SPREAD) -> np.ndarray:
    """Elements of slerp rows whose rounding point a_j = bf16(res_j / na) or
    b_j = bf16(out_j / nb) lies within a relative `delta` (the fp32 spread)
    of a bf16 halfway point: the two ends of the spread round differently."""
    def amb(bits):
        v = wl.bf16_bits_to_f32(bits).astype(np.float64)
        q = v / np.sqrt((v * v).sum(axis=1) + eps)[:, None]
        return oracle.bf16_rne_array(q * (1 - delta)) != oracle.bf16_rne_array(q * (1 + delta))

    return amb(x_bits) | amb(o_bits)


def check_forward(seg, got: torch.Tensor, eps: float, out_dtype: str, rows=None, what="wn_forward"):
    w = seg.w if rows is None else seg.w[rows]
    g = None if seg.g is None else (seg.g if rows is None else seg.g[rows])
    ref = oracle.wn_forward(w, g, rho=seg.radius, eps=eps, nthreads=oracle.default_threads())
    got_h = got if rows is None else got[torch.as_tensor(rows, device=got.device)]
    if out_dtype == "bf16":
        gb = host_bits(got_h)
        ref_bits = oracle.bf16_rne_array(ref)
        lo = oracle.bf16_rne_array(ref - SPREAD * np.abs(ref))
        hi = oracle.bf16_rne_array(ref + SPREAD * np.abs(ref))
        return assert_bf16_rows(gb, ref_bits, lo, hi, what)
    else:
        bad = rel_violations(host_f32(got_h), ref, 2e-6)
        assert not bad.any(), f"{what}: {int(bad.sum())} fp32 outputs beyond 2e-6 relative"


def check_backward(seg, gw: torch.Tensor, gg, eps: float, rows=None, what="wn_backward"):
    sel = slice(None) if rows is None else rows
    w, gy = seg.w[sel], seg.gy[sel]
    g = None if seg.g is None else seg.g[sel]
    ref_w, ref_g = oracle.wn_backward(w, gy, g, rho=seg.radius, eps=eps, nthreads=oracle.default_threads())
    idx = None if rows is None else torch.as_tensor(rows, device=gw.device)
    got_w = host_f32(gw if idx is None else gw[idx])
    gy64 = (wl.bf16_bits_to_f32(gy) if gy.dtype == np.uint16 else gy).astype(np.float64)
    w64 = w.astype(np.float64)
    n = np.sqrt(np.einsum("ij,ij->i", w64, w64) + eps)
    gabs = np.ones(len(w64)) if g is None else np.abs(g.astype(np.float64))
    rms = np.sqrt(np.mean(gy64 ** 2, axis=1))
    floor = (gabs * seg.radius / n * rms)[:, None]
    bad = rel_violations(got_w, ref_w, 1e-5, floor)
    assert not bad.any(), f"{what}: {int(bad.sum())} grad_w entries beyond tolerance " \
                          f"(first at {np.argwhere(bad)[0].tolist()})"
    if g is not None:
        got_g = host_f32(gg if idx is None else gg[idx])
        fl = seg.radius * np.linalg.norm(gy64, axis=1)
        badg = rel_violations(got_g, ref_g, 1e-5, fl)
        assert not badg.any(), f"{what}: {int(badg.sum())} grad_g entries beyond tolerance"


def check_renorm(seg, got: torch.Tensor, eps: float, rows=None, what="row_renorm"):
    w = seg.w if rows is None else seg.w[rows]
    ref = oracle.row_renorm(w, rho=seg.radius, eps=eps, nthreads=oracle.default_threads())
    got_h = host_f32(got if rows is None else got[torch.as_tensor(rows, device=got.device)])
    bad = rel_violations(got_h, ref, 2e-6)
    assert not bad.any(), f"{what}: {int(bad.sum())} fp32 outputs beyond 2e-6 relative"


def _proj_check(got, ref, d, what):
    """The projection's tolerance: 1e-5 relative with a floor of the row's
    RMS of the input (the subtraction d - w D/n^2 can cancel)."""
    d64 = d.astype(np.float64)
    floor = np.sqrt(np.mean(d64 ** 2, axis=1))[:, None]
    bad = rel_violations(got, ref, 1e-5, floor)
    assert not bad.any(), f"{what}: {int(bad.sum())} entries beyond tolerance (first at {np.argwhere(bad)[0].tolist()})"


def check_project(seg, got: torch.Tensor, eps: float, rows=None, what="grad_project", flags=0):
    sel = slice(None) if rows is None else rows
    w, G = seg.w[sel], seg.gy[sel]
    ref = oracle.grad_project(w, G, eps=eps, flags=flags, nthreads=oracle.default_threads())
    got_h = host_f32(got if rows is None else got[torch.as_tensor(rows, device=got.device)])
    _proj_check(got_h, ref, G, what)


def check_momentum(seg, got_w: torch.Tensor, got_m: torch.Tensor, eps: float, rows=None, what="renorm_momentum"):
    sel = slice(None) if rows is None else rows
    w, m = seg.w[sel], seg.gy[sel]
    ref_w, ref_m = oracle.renorm_momentum(w, m, rho=seg.radius, eps=eps, nthreads=oracle.default_threads())
    idx = None if rows is None else torch.as_tensor(rows, device=got_w.device)
    gw = host_f32(got_w if idx is None else got_w[idx])
    gm = host_f32(got_m if idx is None else got_m[idx])
    bad = rel_violations(gw, ref_w, 2e-6)
    assert not bad.any(), f"{what}: {int(bad.sum())} renormed entries beyond 2e-6 relative"
    _proj_check(gm, ref_m, m, what + " (momentum)")


def check_l2(act, got: torch.Tensor, eps: float, residual=True, rows=None, what="l2_rows", flags=0):
    sel = slice(None) if rows is None else rows
    x = act.x[sel]
    r = act.r[sel] if (residual and act.r is not None) else None
    nt = oracle.default_threads()
    ref = oracle.l2_rows(x, r, eps=eps, flags=flags, nthreads=nt)
    lo, hi = oracle.l2_rows_interval(x, r, eps=eps, delta=SPREAD, flags=flags, nthreads=nt)
    gb = host_bits(got if rows is None else got[torch.as_tensor(rows, device=got.device)])
    return assert_bf16_rows(gb, ref, lo, hi, what)


def check_slerp(act, got: torch.Tensor, eps: float, rows=None, what="slerp_rows", flags=0):
    sel = slice(None) if rows is None else rows
    x, o = act.x[sel], act.r[sel]
    nt = oracle.default_threads()
    ref = oracle.slerp_rows(x, o, act.alpha, eps=eps, flags=flags, nthreads=nt)
    lo, hi = oracle.slerp_rows_interval(x, o, act.alpha, eps=eps, delta=SPREAD, flags=flags, nthreads=nt)
    gb = host_bits(got if rows is None else got[torch.as_tensor(rows, device=got.device)])
    return assert_bf16_rows(gb, ref, lo, hi, what, ambiguous=slerp_ambiguous(x, o, eps))


def sample_rows(n: int, k: int, seed: int, must=()) -> np.ndarray:
    """Sorted unique sample of k rows plus the first, the last and `must`."""
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=min(k, n), replace=False).tolist()) | {0, n - 1} | set(int(m) for m in must)
    return np.array(sorted(pick), np.int64)
