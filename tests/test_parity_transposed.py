"""GPU parity of the weight calls on transposed rows (GPT-2's Conv1D keeps
its weight as [in, out], so each unit row -- one output channel -- is a
column of the stored matrix; DragonScale package description, "Supported
layers").  Every result is compared, transposed back, with the float64
oracle applied to the transposed matrix: the same definitions, row by row.
Both kernels are covered: whole column tiles staged over a cluster, and the
column kernel for stored matrices too tall for that."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from l2_row_b200 import ds
from l2_row_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

# (stored rows = in, stored cols = out): GPT-2 small's Conv1D shapes,
# GPT-2 XL's MLP pair ([1600, 6400] and [6400, 1600]: narrow tiles over
# clusters), ragged ones (out not a multiple of 4; one output channel), bands
# whose box heights must be rounded so that every TMA box starts on 128 bytes
# ([13000, 24]: 16-column tiles in boxes of 236 rows; [301, 40]: 32-column
# tiles, a bf16 GY in two boxes), and one too tall for eight CTAs' shared
# memory, which takes the column kernel ([30000, 8])
SHAPES = [(768, 2304), (768, 768), (768, 3072), (3072, 768), (1600, 6400), (6400, 1600), (100, 13), (7, 1),
          (5, 6), (13000, 24), (301, 40), (30000, 8)]


def _stored(rng, K, N, ld_pad=0):
    """fp32 [K, N] rows drifted per output channel (column), in a padded
    [K, N + pad] buffer; returns (host [K, N], device view)."""
    w_t = wl.drifted_rows(rng, N, K, 0.02)            # [N, K]: one row per channel
    host = np.ascontiguousarray(w_t.T)                 # stored [K, N]
    ld = (N + 3) // 4 * 4 + ld_pad
    dev, buf = gu.padded(K, N, ld, torch.float32, gu.CANARY_F32)
    dev.copy_(gu.dev_f32(host))
    return host, dev, buf, ld


def _seg_t(w_host, g, gy_host, radius=1.0):
    """The row-major (unit rows = output channels) view the oracle takes."""
    return wl.WeightSeg("t", np.ascontiguousarray(w_host.T), g,
                        None if gy_host is None else np.ascontiguousarray(gy_host.T), radius=radius)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_forward(out_dtype):
    rng = np.random.default_rng(91)
    for K, N in SHAPES:
        w, wd, _, ld = _stored(rng, K, N, ld_pad=4)
        g = wl.gains(rng, N)
        dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        canary = gu.CANARY_BF16 if out_dtype == "bf16" else gu.CANARY_F32
        ld_o = (N + 7) // 8 * 8 + 8          # rows of W_eff start on 16 bytes in either dtype
        o, obuf = gu.padded(K, N, ld_o, dt, canary)
        ds.ds_wn_forward([ds.WSeg(w=wd, gain=gu.dev_f32(g), w_eff=o, transposed=True)], out_dtype, 1e-6)
        torch.cuda.synchronize()
        assert gu.guards_intact(obuf, K, N, ld_o, canary), (K, N)
        gu.check_forward(_seg_t(w, g, None), o.t().contiguous(), 1e-6, out_dtype, what=f"fwd [{K},{N}]")


@pytest.mark.parametrize("gy_dtype", ["bf16", "f32"])
def test_backward(gy_dtype):
    rng = np.random.default_rng(92)
    for K, N in SHAPES:
        w, wd, _, ld = _stored(rng, K, N)
        g = wl.gains(rng, N)
        gy = rng.standard_normal((K, N)).astype(np.float32) * np.float32(1e-3)
        if gy_dtype == "bf16":
            gy = wl.to_bf16_bits(gy)
        ld_g = (N + 7) // 8 * 8                # rows of GY start on 16 bytes
        gyd, _ = gu.padded(K, N, ld_g, torch.bfloat16 if gy_dtype == "bf16" else torch.float32,
                           gu.CANARY_BF16 if gy_dtype == "bf16" else gu.CANARY_F32)
        gyd.copy_(gu.dev_bf16(gy) if gy_dtype == "bf16" else gu.dev_f32(gy))
        gw, gwbuf = gu.padded(K, N, ld, torch.float32, gu.CANARY_F32)
        gg = torch.empty(N, dtype=torch.float32, device="cuda")
        ds.ds_wn_backward([ds.WSeg(w=wd, gain=gu.dev_f32(g), gy=gyd, grad_w=gw, grad_g=gg, transposed=True)],
                          gy_dtype, 1e-6)
        torch.cuda.synchronize()
        assert gu.guards_intact(gwbuf, K, N, ld, gu.CANARY_F32), (K, N)
        gu.check_backward(_seg_t(w, g, gy), gw.t().contiguous(), gg, 1e-6, what=f"bwd [{K},{N}]")


def test_renorm_and_projections():
    rng = np.random.default_rng(93)
    for K, N in SHAPES:
        w, wd, _, ld = _stored(rng, K, N)
        G = rng.standard_normal((K, N)).astype(np.float32)
        # renorm in place
        ds.ds_row_renorm([ds.WSeg(w=wd, transposed=True)], 1e-6)
        torch.cuda.synchronize()
        gu.check_renorm(_seg_t(w, None, None), wd.t().contiguous(), 1e-6, what=f"renorm [{K},{N}]")
        # gradient projection
        w2, wd2, _, _ = _stored(rng, K, N)
        Gd, _ = gu.padded(K, N, ld, torch.float32, gu.CANARY_F32)
        Gd.copy_(gu.dev_f32(G))
        ds.ds_grad_project([ds.WSeg(w=wd2, grad_w=Gd, transposed=True)], 1e-6)
        torch.cuda.synchronize()
        gu.check_project(_seg_t(w2, None, G), Gd.t().contiguous(), 1e-6, what=f"project [{K},{N}]")
        # momentum projection + renorm
        md, _ = gu.padded(K, N, ld, torch.float32, gu.CANARY_F32)
        md.copy_(gu.dev_f32(G))
        ds.ds_renorm_momentum([ds.WSeg(w=wd2, grad_w=md, transposed=True)], 1e-6)
        torch.cuda.synchronize()
        gu.check_momentum(_seg_t(w2, None, G), wd2.t().contiguous(), md.t().contiguous(), 1e-6,
                          what=f"momentum [{K},{N}]")


def test_mixed_table_and_scalar_gain():
    """A table mixing normal and transposed segments in one call; a scalar
    gain on a transposed segment."""
    rng = np.random.default_rng(94)
    K, N = 768, 2304
    w, wd, _, _ = _stored(rng, K, N)
    gy = wl.to_bf16_bits(rng.standard_normal((K, N)).astype(np.float32) * np.float32(1e-3))
    row = wl.WeightSeg("r", wl.drifted_rows(rng, 64, 768, 0.02), wl.gains(rng, 64),
                       wl.to_bf16_bits(rng.standard_normal((64, 768)).astype(np.float32)))
    gs = torch.full((1,), 0.75, dtype=torch.float32, device="cuda")
    gw_t = torch.empty(K, N, dtype=torch.float32, device="cuda")
    gg_t = torch.empty(N + 1, dtype=torch.float32, device="cuda")
    gw_r = torch.empty(64, 768, dtype=torch.float32, device="cuda")
    gg_r = torch.empty(64, dtype=torch.float32, device="cuda")
    before = ds.ds_launch_count()
    ds.ds_wn_backward([ds.WSeg(w=gu.dev_f32(row.w), gain=gu.dev_f32(row.g), gy=gu.dev_bf16(row.gy), grad_w=gw_r,
                               grad_g=gg_r),
                       ds.WSeg(w=wd, gain=gs, gy=gu.dev_bf16(gy), grad_w=gw_t, grad_g=gg_t, transposed=True,
                               gain_scalar=True)], "bf16", 1e-6)
    torch.cuda.synchronize()
    assert ds.ds_launch_count() - before == 3          # rows, transposed rows, the gain sum
    gu.check_backward(row, gw_r, gg_r, 1e-6, what="row segment")
    seg = _seg_t(w, np.full(N, 0.75, np.float32), gy)
    gu.check_backward(seg, gw_t.t().contiguous(), gg_t[:N], 1e-6, what="transposed, scalar gain")
    h = gu.host_f32(gg_t)
    assert abs(float(h[N]) - float(np.sum(h[:N], dtype=np.float64))) <= np.spacing(np.float32(abs(h[N])))


@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_extreme_columns(eps):
    """Column tiles whose fp32 sums overflow (|w| ~ 1e25), or at eps = 0 fall
    below 2^-100 (|w| ~ 1e-30), take the exact pass; a tile of ordinary
    columns beside them keeps the fp32 pass.  Both against the oracle."""
    rng = np.random.default_rng(95)
    K, N = 768, 384
    w, wd, _, ld = _stored(rng, K, N)
    w[:, 5] *= np.float32(1e27)          # tile 0: one overflowing column
    w[:, 200] *= np.float32(1e-28)       # a later tile: one tiny column
    wd.copy_(gu.dev_f32(w))
    g = wl.gains(rng, N)
    for out_dtype in ("f32", "bf16"):
        dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        o = torch.empty(K, N, dtype=dt, device="cuda")
        ds.ds_wn_forward([ds.WSeg(w=wd, gain=gu.dev_f32(g), w_eff=o, transposed=True)], out_dtype, eps)
        torch.cuda.synchronize()
        gu.check_forward(_seg_t(w, g, None), o.t().contiguous(), eps, out_dtype, what=f"extreme fwd {out_dtype}")
    gy = wl.to_bf16_bits(rng.standard_normal((K, N)).astype(np.float32) * np.float32(1e-3))
    gw = torch.empty(K, N, dtype=torch.float32, device="cuda")
    gg = torch.empty(N, dtype=torch.float32, device="cuda")
    gyd = torch.empty(K, N, dtype=torch.bfloat16, device="cuda")
    gyd.copy_(gu.dev_bf16(gy))
    ds.ds_wn_backward([ds.WSeg(w=wd, gain=gu.dev_f32(g), gy=gyd, grad_w=gw, grad_g=gg, transposed=True)],
                      "bf16", eps)
    torch.cuda.synchronize()
    gu.check_backward(_seg_t(w, g, gy), gw.t().contiguous(), gg, eps, what="extreme bwd")
    ds.ds_row_renorm([ds.WSeg(w=wd, transposed=True)], eps)
    torch.cuda.synchronize()
    gu.check_renorm(_seg_t(w, None, None), wd.t().contiguous(), eps, what="extreme renorm")


# ConvTranspose weights [in, out, k...] stored [in, out * G] (G = the kernel's
# volume): unit row r = the G columns [r G, r G + G) of every stored row.
# (in, out, G): ConvTranspose2d 3x3, ConvTranspose1d k=4, ConvTranspose3d
# 3x3x3, a ragged one, a 4x4 decoder layer, the largest G, G >= 64 (one unit
# row per block), ConvTranspose3d 2x2x2 with a ragged out, and a 2x2 layer too
# tall for the column tiles.  Powers of two up to 32 take the column tiles
# (whole unit rows per tile), the rest the grouped kernel.
GROUPED = [(64, 32, 9), (128, 64, 4), (16, 8, 27), (5, 7, 6), (512, 256, 16), (3, 2, 256), (40, 3, 130),
           (96, 13, 8), (14000, 6, 4)]


def _unit_rows(stored: np.ndarray, G: int) -> np.ndarray:
    """[in, out * G] -> the unit rows [out, in * G] (stored row j's G
    elements of unit row r at j G .. j G + G - 1)."""
    K, N = stored.shape
    return np.ascontiguousarray(stored.reshape(K, N // G, G).transpose(1, 0, 2).reshape(N // G, K * G))


def _dev_unit_rows(t: torch.Tensor, G: int) -> torch.Tensor:
    K, N = t.shape
    return t.reshape(K, N // G, G).permute(1, 0, 2).reshape(N // G, K * G).contiguous()


def _grouped(rng, K, R, G):
    """Weights drifted per output channel, stored [K, R G]."""
    units = wl.drifted_rows(rng, R, K * G, 0.02)                     # [R, K G]
    return np.ascontiguousarray(units.reshape(R, K, G).transpose(1, 0, 2).reshape(K, R * G))


def _ld(n: int) -> int:
    """A leading dimension >= n whose rows start on 16 bytes in fp32 and bf16."""
    return (n + 7) // 8 * 8


def _dev(a: np.ndarray, ld: int, bf16=False):
    """a (fp32, or bf16 bits) in a [K, ld] device buffer with guard rows;
    returns (view, buffer, canary)."""
    K, N = a.shape
    dt, canary = (torch.bfloat16, gu.CANARY_BF16) if bf16 else (torch.float32, gu.CANARY_F32)
    v, buf = gu.padded(K, N, ld, dt, canary)
    v.copy_(gu.dev_bf16(a) if bf16 else gu.dev_f32(a))
    return v, buf, canary


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_grouped_forward(out_dtype):
    rng = np.random.default_rng(96)
    for K, R, G in GROUPED:
        w = _grouped(rng, K, R, G)
        g = wl.gains(rng, R)
        ld = _ld(R * G)
        wd, _, _ = _dev(w, ld)
        dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        canary = gu.CANARY_BF16 if out_dtype == "bf16" else gu.CANARY_F32
        ld_o = ld + 8
        o, obuf = gu.padded(K, R * G, ld_o, dt, canary)
        ds.ds_wn_forward([ds.WSeg(w=wd, gain=gu.dev_f32(g), w_eff=o, transposed=True, tgroup=G)], out_dtype, 1e-6)
        torch.cuda.synchronize()
        assert gu.guards_intact(obuf, K, R * G, ld_o, canary), (K, R, G)
        seg = wl.WeightSeg("g", _unit_rows(w, G), g, None)
        gu.check_forward(seg, _dev_unit_rows(o, G), 1e-6, out_dtype, what=f"grouped fwd [{K},{R}x{G}]")


@pytest.mark.parametrize("gy_dtype", ["bf16", "f32"])
def test_grouped_backward(gy_dtype):
    rng = np.random.default_rng(97)
    for K, R, G in GROUPED:
        w = _grouped(rng, K, R, G)
        g = wl.gains(rng, R)
        gy = rng.standard_normal((K, R * G)).astype(np.float32) * np.float32(1e-3)
        if gy_dtype == "bf16":
            gy = wl.to_bf16_bits(gy)
        ld = _ld(R * G)
        wd, _, _ = _dev(w, ld)
        gyd, _, _ = _dev(gy, ld, bf16=gy_dtype == "bf16")
        gw, gwbuf = gu.padded(K, R * G, ld, torch.float32, gu.CANARY_F32)
        gg = torch.empty(R, dtype=torch.float32, device="cuda")
        ds.ds_wn_backward([ds.WSeg(w=wd, gain=gu.dev_f32(g), gy=gyd, grad_w=gw, grad_g=gg, transposed=True,
                                   tgroup=G)], gy_dtype, 1e-6)
        torch.cuda.synchronize()
        assert gu.guards_intact(gwbuf, K, R * G, ld, gu.CANARY_F32), (K, R, G)
        seg = wl.WeightSeg("g", _unit_rows(w, G), g, _unit_rows(gy, G))
        gu.check_backward(seg, _dev_unit_rows(gw, G), gg, 1e-6, what=f"grouped bwd [{K},{R}x{G}]")


def test_grouped_renorm_projections_and_scalar_gain():
    rng = np.random.default_rng(98)
    for K, R, G in GROUPED:
        ld = _ld(R * G)
        w = _grouped(rng, K, R, G)
        wd, wbuf, can = _dev(w, ld)
        ds.ds_row_renorm([ds.WSeg(w=wd, transposed=True, tgroup=G)], 1e-6)
        torch.cuda.synchronize()
        assert gu.guards_intact(wbuf, K, R * G, ld, can), (K, R, G)
        gu.check_renorm(wl.WeightSeg("g", _unit_rows(w, G), None, None), _dev_unit_rows(wd, G), 1e-6,
                        what=f"grouped renorm [{K},{R}x{G}]")
        w2 = _grouped(rng, K, R, G)
        G2 = rng.standard_normal((K, R * G)).astype(np.float32)
        wd2, _, _ = _dev(w2, ld)
        Gd, _, _ = _dev(G2, ld)
        ds.ds_grad_project([ds.WSeg(w=wd2, grad_w=Gd, transposed=True, tgroup=G)], 1e-6)
        torch.cuda.synchronize()
        seg2 = wl.WeightSeg("g", _unit_rows(w2, G), None, _unit_rows(G2, G))
        gu.check_project(seg2, _dev_unit_rows(Gd, G), 1e-6, what=f"grouped project [{K},{R}x{G}]")
        md, _, _ = _dev(G2, ld)
        ds.ds_renorm_momentum([ds.WSeg(w=wd2, grad_w=md, transposed=True, tgroup=G)], 1e-6)
        torch.cuda.synchronize()
        gu.check_momentum(seg2, _dev_unit_rows(wd2, G), _dev_unit_rows(md, G), 1e-6,
                          what=f"grouped momentum [{K},{R}x{G}]")
    # one gain for the whole layer: per-row parts, then their sum
    K, R, G = 64, 32, 9
    ld = _ld(R * G)
    w = _grouped(rng, K, R, G)
    gy = wl.to_bf16_bits(rng.standard_normal((K, R * G)).astype(np.float32) * np.float32(1e-3))
    wd, _, _ = _dev(w, ld)
    gyd, _, _ = _dev(gy, ld, bf16=True)
    gw, _ = gu.padded(K, R * G, ld, torch.float32, gu.CANARY_F32)
    gg = torch.empty(R + 1, dtype=torch.float32, device="cuda")
    gs = torch.full((1,), 0.75, dtype=torch.float32, device="cuda")
    ds.ds_wn_backward([ds.WSeg(w=wd, gain=gs, gy=gyd, grad_w=gw, grad_g=gg, transposed=True, tgroup=G,
                               gain_scalar=True)], "bf16", 1e-6)
    torch.cuda.synchronize()
    seg = wl.WeightSeg("g", _unit_rows(w, G), np.full(R, 0.75, np.float32), _unit_rows(gy, G))
    gu.check_backward(seg, _dev_unit_rows(gw, G), gg[:R], 1e-6, what="grouped, scalar gain")
    h = gu.host_f32(gg)
    assert abs(float(h[R]) - float(np.sum(h[:R], dtype=np.float64))) <= np.spacing(np.float32(abs(h[R])))


@pytest.mark.parametrize("eps", [1e-6, 0.0])
@pytest.mark.parametrize("G", [9, 16])
def test_grouped_extreme_channels(eps, G):
    """ConvTranspose channels whose fp32 sums overflow (|w| ~ 1e25) or, at
    eps = 0, fall below 2^-100 (|w| ~ 1e-30) take the double pass; the other
    blocks keep fp32 (G = 9: the grouped kernel; G = 16: column tiles of whole
    unit rows).  Against the oracle."""
    rng = np.random.default_rng(99)
    K, R = 64, 32
    ld = _ld(R * G)
    w = _grouped(rng, K, R, G)
    w[:, 2 * G:3 * G] *= np.float32(1e27)          # channel 2
    w[:, 20 * G:21 * G] *= np.float32(1e-28)       # channel 20, another block
    g = wl.gains(rng, R)
    for out_dtype in ("f32", "bf16"):
        wd, _, _ = _dev(w, ld)
        dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        o = torch.empty(K, ld, dtype=dt, device="cuda")[:, :R * G]
        ds.ds_wn_forward([ds.WSeg(w=wd, gain=gu.dev_f32(g), w_eff=o, transposed=True, tgroup=G)], out_dtype, eps)
        torch.cuda.synchronize()
        gu.check_forward(wl.WeightSeg("g", _unit_rows(w, G), g, None), _dev_unit_rows(o, G), eps, out_dtype,
                         what=f"grouped extreme fwd {out_dtype}")
    gy = wl.to_bf16_bits(rng.standard_normal((K, R * G)).astype(np.float32) * np.float32(1e-3))
    wd, _, _ = _dev(w, ld)
    gyd, _, _ = _dev(gy, ld, bf16=True)
    gw, _ = gu.padded(K, R * G, ld, torch.float32, gu.CANARY_F32)
    gg = torch.empty(R, dtype=torch.float32, device="cuda")
    ds.ds_wn_backward([ds.WSeg(w=wd, gain=gu.dev_f32(g), gy=gyd, grad_w=gw, grad_g=gg, transposed=True, tgroup=G)],
                      "bf16", eps)
    torch.cuda.synchronize()
    gu.check_backward(wl.WeightSeg("g", _unit_rows(w, G), g, _unit_rows(gy, G)), _dev_unit_rows(gw, G), gg, eps,
                      what="grouped extreme bwd")
    ds.ds_row_renorm([ds.WSeg(w=wd, transposed=True, tgroup=G)], eps)
    torch.cuda.synchronize()
    gu.check_renorm(wl.WeightSeg("g", _unit_rows(w, G), None, None), _dev_unit_rows(wd, G), eps,
                    what="grouped extreme renorm")
