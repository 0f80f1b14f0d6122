"""The no-alloc slerp backward entry point, ds_slerp_rows_backward_noalloc.

It serves callers that cannot allocate device memory where they run the
backward (a runtime whose device memory all belongs to its own pool, or code
that must not risk the device-wide synchronisation of cudaMalloc / cudaFree)
and so cannot hand ds_slerp_rows_backward a workspace: dalpha's partial sums
go to a 64 MB static device array built into the library instead.  The pages
have no counterpart.  Its results must be bitwise those of
ds_slerp_rows_backward with a caller workspace, call after call (the array is
shared and keeps the previous call's contents), and rows whose partial sums
need more than the array holds must be refused.

This file is collected last (test_zz_...), so a run that stops at the first
failure has run every other test before it.
"""
from __future__ import annotations

import ctypes as ct

import numpy as np
import pytest
import torch

from l2_row_b200 import ds
from l2_row_b200 import workloads as wl


def test_noalloc_symbol_exported_and_declared():
    assert "ds_slerp_rows_backward_noalloc" in ds.EXPORTS
    assert hasattr(ds.lib(), "ds_slerp_rows_backward_noalloc")


def test_noalloc_host_validation_without_gpu():
    """Bad arguments fail on the host before any launch (no GPU needed)."""
    B = 0x7F0000000000
    seg = ds.ds_agseg(x=B, r=B + (1 << 30), dy=B + (2 << 30), dx=B + (3 << 30), dr=B + (4 << 30),
                      alpha=B + (5 << 30), rows=4, cols=8, ld=8, ld_d=8)
    arr = (ds.ds_agseg * 1)(seg)
    before = ds.ds_launch_count()
    bad = ds.ds_agseg(x=B, r=0, dy=B + (2 << 30), dx=B + (3 << 30), dr=B + (4 << 30), alpha=B + (5 << 30),
                      rows=4, cols=8, ld=8, ld_d=8)
    assert ds.lib().ds_slerp_rows_backward_noalloc((ds.ds_agseg * 1)(bad), 1, ct.c_float(1e-6), None, None) == \
        ds.DS_ERR_INVALID_ARG                                   # out (r) required
    assert ds.lib().ds_slerp_rows_backward_noalloc(arr, 1, ct.c_float(-1.0), None, None) == ds.DS_ERR_INVALID_ARG
    empty = ds.ds_agseg(x=0, r=0, dy=0, dx=0, dr=0, alpha=B, rows=0, cols=8, ld=8, ld_d=8)
    assert ds.lib().ds_slerp_rows_backward_noalloc((ds.ds_agseg * 1)(empty), 1, ct.c_float(1e-6), None, None) == \
        ds.DS_OK
    assert ds.ds_launch_count() == before


def _run(res, out, alpha, dh, noalloc):
    R, C = res.shape
    dres = torch.empty(R, C, dtype=torch.float32, device="cuda")
    dout = torch.empty_like(dres)
    da = torch.empty(C, dtype=torch.float32, device="cuda")
    seg = ds.AGSeg(x=torch.from_numpy(res.view(np.int16)).cuda().view(torch.bfloat16),
                   r=torch.from_numpy(out.view(np.int16)).cuda().view(torch.bfloat16),
                   dy=torch.from_numpy(dh.view(np.int16)).cuda().view(torch.bfloat16),
                   dx=dres, dr=dout, alpha=torch.from_numpy(alpha).cuda())
    if noalloc:
        ds.ds_slerp_rows_backward_noalloc([seg], 1e-6, dalpha=da)
    else:
        ds.ds_slerp_rows_backward([seg], 1e-6, dalpha=da)
    torch.cuda.synchronize()
    return dres, dout, da


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(300, 1024), (2048, 4096), (64, 7168)])
def test_noalloc_matches_workspace_bitwise(shape):
    rng = np.random.default_rng(91)
    res, out, dh = (wl.normal_bf16(rng, shape) for _ in range(3))
    alpha = wl.alpha_vec(rng, shape[1])
    a = _run(res, out, alpha, dh, noalloc=False)
    b = _run(res, out, alpha, dh, noalloc=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = _run(res, out, alpha, dh, noalloc=True)   # the scratch is reused: same bits again
    assert torch.equal(b[2], c[2])


SCRATCH_BYTES = 64 << 20   # the built-in array


def widest_accepted_cols() -> int:
    """The widest row (a multiple of 8) whose dalpha partial sums fit the
    built-in array on this device (8,712 on a 148-SM B200)."""
    c = 8
    while ds.ds_slerp_rows_backward_workspace(c + 8) <= SCRATCH_BYTES:
        c += 8
    return c


@pytest.mark.gpu
def test_noalloc_widest_accepted_rows_match_workspace_bitwise():
    C = widest_accepted_cols()
    assert ds.ds_slerp_rows_backward_workspace(C) <= SCRATCH_BYTES < ds.ds_slerp_rows_backward_workspace(C + 8)
    rng = np.random.default_rng(93)
    res, out, dh = (wl.normal_bf16(rng, (600, C)) for _ in range(3))
    alpha = wl.alpha_vec(rng, C)
    a = _run(res, out, alpha, dh, noalloc=False)
    for _ in range(2):
        b = _run(res, out, alpha, dh, noalloc=True)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


@pytest.mark.gpu
def test_noalloc_refuses_rows_wider_than_its_scratch():
    rng = np.random.default_rng(92)
    C = widest_accepted_cols() + 8
    res, out, dh = (wl.normal_bf16(rng, (4, C)) for _ in range(3))
    with pytest.raises(ds.DSError) as e:
        _run(res, out, wl.alpha_vec(rng, C), dh, noalloc=True)
    assert e.value.status == ds.DS_ERR_INVALID_ARG
    assert "built-in scratch" in ds.ds_last_error()
