"""The no-alloc slerp backward entry point (a convenience of this library;
the pages have no counterpart): dalpha's partial sums go to a scratch array
built into the library instead of a caller workspace.  Its results must be
bitwise those of ds_slerp_rows_backward with a workspace."""
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


@pytest.mark.gpu
def test_noalloc_refuses_rows_wider_than_its_scratch():
    rng = np.random.default_rng(92)
    C = 8720  # dalpha lines of 8,720 columns on 148 SMs need more than the 64 MB scratch
    res, out, dh = (wl.normal_bf16(rng, (4, C)) for _ in range(3))
    with pytest.raises(ds.DSError):
        _run(res, out, wl.alpha_vec(rng, C), dh, noalloc=True)
