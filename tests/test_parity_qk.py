"""GPU parity of Dory's q and k rows (TensorFold PR #1260, tf_qk_rows_l2)
against the float64 oracle: every q and k output within 1 bf16 ulp of the
oracle's point value or inside its interval (cosf's ulps on the fp32 angle,
the rotation's fp32 steps), v copied bit for bit, cache rows by slot, on the
pages' workload (head dim 256, 16 query heads over 4, a third of the rows
past position 199,800) and on other head sizes, ragged row counts and
padded leading dimensions."""
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


def _dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


def run(w: wl.QKRows, eps=1e-6, scale=True, slot=None, cache_rows=None, ld_pad=0, with_v=True):
    """Run ds_qk_rows_l2 on w; returns (q_out, k_cache, v_cache) host bits
    (caches [cache_rows, hk*D]) and the guard check of the padded buffers."""
    R, D = w.rows, w.head_dim
    wq, wk = w.hq * D, w.hk * D
    cache_rows = R if cache_rows is None else cache_rows
    ldq, ldk = wq + ld_pad, wk + ld_pad
    q, qbuf = gu.padded(R, wq, ldq, torch.bfloat16, gu.CANARY_BF16) if wq else (None, None)
    k, _ = gu.padded(R, wk, ldk, torch.bfloat16, gu.CANARY_BF16) if wk else (None, None)
    v, _ = gu.padded(R, wk, ldk, torch.bfloat16, gu.CANARY_BF16) if wk and with_v else (None, None)
    if q is not None:
        q.copy_(gu.dev_bf16(w.q))
    if k is not None:
        k.copy_(gu.dev_bf16(w.k))
    if v is not None:
        v.copy_(gu.dev_bf16(w.v))
    qo, qobuf = gu.padded(R, wq, ldq, torch.bfloat16, gu.CANARY_BF16) if wq else (None, None)
    kc, kcbuf = gu.padded(cache_rows, wk, ldk, torch.bfloat16, gu.CANARY_BF16) if wk else (None, None)
    vc, vcbuf = gu.padded(cache_rows, wk, ldk, torch.bfloat16, gu.CANARY_BF16) if wk and with_v else (None, None)
    seg = ds.QKSeg(head_dim=D, pos=_dev_i32(w.pos), inv_freq=gu.dev_f32(w.inv), q=q, q_out=qo, k=k, k_cache=kc,
                   v=v, v_cache=vc, slot=None if slot is None else _dev_i32(slot),
                   q_scale=gu.dev_f32(w.q_scale) if scale and wq else None)
    ds.ds_qk_rows_l2([seg], eps)
    torch.cuda.synchronize()
    guards = True
    if qo is not None:
        guards &= gu.guards_intact(qobuf, R, wq, ldq, gu.CANARY_BF16)
    if kc is not None:
        guards &= gu.guards_intact(kcbuf, cache_rows, wk, ldk, gu.CANARY_BF16)
    if vc is not None:
        guards &= gu.guards_intact(vcbuf, cache_rows, wk, ldk, gu.CANARY_BF16)
    host = lambda t: None if t is None else gu.host_bits(t)
    return host(qo), host(kc), host(vc), guards


def check(w: wl.QKRows, qo, ko, eps=1e-6, scale=True, flags=0, rows=None, what=""):
    sel = slice(None) if rows is None else rows
    nt = oracle.default_threads()
    sc = w.q_scale if scale else None
    qr, kr = oracle.qk_rows_l2(w.q[sel], w.k[sel], w.pos[sel], w.inv, sc, head_dim=w.head_dim, eps=eps,
                               flags=flags, nthreads=nt)
    ql, qh, kl, kh = oracle.qk_rows_l2_interval(w.q[sel], w.k[sel], w.pos[sel], w.inv, sc, head_dim=w.head_dim,
                                                eps=eps, flags=flags, nthreads=nt)
    if w.hq:
        gu.assert_bf16_rows(qo[sel], qr, ql, qh, what + " q", ambiguous=gu.interval_admits_beyond_ulp(qr, ql, qh))
    if w.hk:
        gu.assert_bf16_rows(ko[sel], kr, kl, kh, what + " k", ambiguous=gu.interval_admits_beyond_ulp(kr, kl, kh))


def test_dory_heads_all_rows():
    w = wl.qk_rows(31, rows=96)
    qo, kc, vc, guards = run(w)
    assert guards
    check(w, qo, kc, what="dory")
    assert np.array_equal(vc, w.v)


# (512, 32, 4): 40 heads of 512 per row, tasks in two rounds per warp
@pytest.mark.parametrize("D,hq,hk", [(16, 3, 1), (32, 2, 2), (64, 8, 2), (128, 5, 3), (512, 2, 1), (256, 1, 0),
                                     (256, 0, 3), (512, 32, 4)])
def test_head_sizes_ragged_rows_padded(D, hq, hk):
    for rows in (1, 2, 7, 33):
        w = wl.qk_rows(32 + D + rows, rows=rows, head_dim=D, hq=hq, hk=hk)
        for eps in (1e-6, 0.0):
            qo, kc, vc, guards = run(w, eps=eps, ld_pad=8)
            assert guards, (D, hq, hk, rows)
            check(w, qo, kc, eps=eps, what=f"D={D} hq={hq} hk={hk} rows={rows} eps={eps}")
            if hk:
                assert np.array_equal(vc, w.v)


def test_no_scale_and_no_v():
    w = wl.qk_rows(40, rows=20)
    qo, kc, vc, guards = run(w, scale=False, with_v=False)
    assert guards and vc is None
    check(w, qo, kc, scale=False, what="no scale")


def test_cache_slots():
    """Rows go to the cache rows their slots name (here reversed into a
    larger ring); untouched cache rows keep their canaries."""
    w = wl.qk_rows(41, rows=24)
    cache_rows = 64
    slot = (np.arange(24)[::-1] * 2 + 5).astype(np.int32)
    qo, kc, vc, guards = run(w, slot=slot, cache_rows=cache_rows)
    assert guards
    check(w, qo, kc[slot], what="slots")
    assert np.array_equal(vc[slot], w.v)
    others = np.setdiff1d(np.arange(cache_rows), slot)
    assert np.all(kc[others] == gu.CANARY_BF16) and np.all(vc[others] == gu.CANARY_BF16)


def test_bad_slot_is_reported_and_skipped():
    w = wl.qk_rows(42, rows=8, head_dim=64, hq=2, hk=1)
    slot = np.arange(8, dtype=np.int32)
    slot[3] = 99                        # past the cache
    qo, kc, vc, _ = run(w, slot=slot, cache_rows=8)
    assert ds.ds_get_device_status() == ds.DS_ERR_INVALID_ARG
    assert ds.ds_get_device_status() == ds.DS_OK          # read and cleared
    ok = slot != 99
    qr, kr = oracle.qk_rows_l2(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=64)
    ql, qh, kl, kh = oracle.qk_rows_l2_interval(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=64)
    gu.assert_bf16_rows(qo, qr, ql, qh, "q rows are all written", ambiguous=gu.interval_admits_beyond_ulp(qr, ql, qh))
    gu.assert_bf16_rows(kc[slot[ok]], kr[ok], kl[ok], kh[ok], "k rows with good slots",
                        ambiguous=gu.interval_admits_beyond_ulp(kr[ok], kl[ok], kh[ok]))
    assert np.all(kc[3] == gu.CANARY_BF16)     # row 3's slot 99 wrote nothing; cache row 3 is nobody's


def test_in_place():
    w = wl.qk_rows(43, rows=16, head_dim=128, hq=4, hk=2)
    ref_q, ref_k, ref_v, _ = run(w)
    D = 128
    q, k, v = gu.dev_bf16(w.q), gu.dev_bf16(w.k), gu.dev_bf16(w.v)
    seg = ds.QKSeg(head_dim=D, pos=_dev_i32(w.pos), inv_freq=gu.dev_f32(w.inv), q=q, q_out=q, k=k, k_cache=k,
                   v=v, v_cache=v, q_scale=gu.dev_f32(w.q_scale))
    ds.ds_qk_rows_l2([seg])
    torch.cuda.synchronize()
    assert np.array_equal(gu.host_bits(q), ref_q)
    assert np.array_equal(gu.host_bits(k), ref_k)
    assert np.array_equal(gu.host_bits(v), ref_v)


def test_position_zero():
    """No rotation (every angle 0): each head is its own l2 row."""
    w = wl.qk_rows(44, rows=32, head_dim=256, hq=4, hk=2)
    w.pos[:] = 0
    qo, kc, _, _ = run(w, scale=False)
    check(w, qo, kc, scale=False, what="pos 0")


def test_controls_are_detected():
    w = wl.qk_rows(45, rows=48)
    qo, kc, _, _ = run(w)
    check(w, qo, kc)
    nt = oracle.default_threads()
    for fl in (oracle.OR_DROP_ROT, oracle.OR_DROP_QNORM):
        ql, qh, kl, kh = oracle.qk_rows_l2_interval(w.q, w.k, w.pos, w.inv, w.q_scale, head_dim=256, flags=fl,
                                                    nthreads=nt)
        assert bf16_interval_violations(qo, ql, qh).any(), hex(fl)


def test_extreme_heads_rescale():
    """Heads whose fp32 sum of squares overflows (|x| ~ 1e30) or, at eps = 0,
    underflows (|x| ~ 1e-30) take the exact power-of-two rescale."""
    for scale, eps in ((1e30, 1e-6), (1e-30, 0.0)):
        w = wl.qk_rows(46, rows=6, head_dim=128, hq=2, hk=2)
        w.q = wl.to_bf16_bits((wl.bf16_bits_to_f32(w.q) * np.float32(scale)).astype(np.float32))
        w.k = wl.to_bf16_bits((wl.bf16_bits_to_f32(w.k) * np.float32(scale)).astype(np.float32))
        qo, kc, _, _ = run(w, eps=eps)
        check(w, qo, kc, eps=eps, what=f"scale {scale}")


def test_sampled_rows_at_bench_size():
    """The bench's shape and launch ([16384 rows] of Dory's heads), checked on
    sampled rows of both position ranges."""
    w = wl.qk_rows(0, rows=16384)
    qo, kc, vc, _ = run(w)
    rows = gu.sample_rows(16384, 48, 47, must=(0, 16383, 10922, 10923))
    check(w, qo, kc, rows=rows, what="bench size")
    assert np.array_equal(vc, w.v)


def test_segments_of_several_head_sizes_in_one_call():
    """A table mixing head sizes runs one launch per head size; every
    segment matches the oracle."""
    ws = [wl.qk_rows(50 + i, rows=r, head_dim=D, hq=hq, hk=hk)
          for i, (r, D, hq, hk) in enumerate([(9, 64, 4, 2), (5, 256, 2, 1), (7, 64, 2, 2), (3, 128, 1, 1)])]
    segs, outs = [], []
    for w in ws:
        q, k, v = gu.dev_bf16(w.q), gu.dev_bf16(w.k), gu.dev_bf16(w.v)
        qo, kc, vc = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        segs.append(ds.QKSeg(head_dim=w.head_dim, pos=_dev_i32(w.pos), inv_freq=gu.dev_f32(w.inv), q=q, q_out=qo,
                             k=k, k_cache=kc, v=v, v_cache=vc, q_scale=gu.dev_f32(w.q_scale)))
        outs.append((qo, kc, vc))
    before = ds.ds_launch_count()
    ds.ds_qk_rows_l2(segs)
    torch.cuda.synchronize()
    assert ds.ds_launch_count() - before == 3          # head sizes 64, 128, 256
    for w, (qo, kc, vc) in zip(ws, outs):
        check(w, gu.host_bits(qo), gu.host_bits(kc), what=f"D={w.head_dim}")
        assert np.array_equal(gu.host_bits(vc), w.v)
