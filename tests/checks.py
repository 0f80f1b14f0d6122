"""Comparison rules shared by the parity tests.

* bf16 outputs: the GPU bits and the oracle's bits differ by at most 1 in the
  monotone integer order of bf16 patterns (+0 == -0); NaN must meet NaN.
* sharp bf16 check (TensorFold's "range over the fp32 run's spread"): the GPU
  bits lie between the oracle interval form's lo and hi bits.
* fp32 outputs: elementwise relative error against the f64 value.
"""
from __future__ import annotations

import numpy as np

# Relative spread of one fp32 evaluation of a row step on the GPU.  A sum of
# positive terms in a reduction tree of depth d has relative error below
# d * 2^-24 (first order); the deepest tree here (per-thread chains of up to
# 128 terms, 5 shuffle levels, up to 8 warps and 8 CTAs) keeps d below 160, so
# the row norm carries < 4.8e-6 and the scaled output < 5e-6 after the square
# root, reciprocal and product.  1e-5 bounds that with margin while staying
# ~400x tighter than half a bf16 ulp (2^-9).
SPREAD = 1e-5


def bf16_key(bits) -> np.ndarray:
    b = np.asarray(bits).astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_isnan(bits) -> np.ndarray:
    b = np.asarray(bits).astype(np.int32)
    return (b & 0x7FFF) > 0x7F80


def bf16_ulp_violations(got, want, max_ulp: int = 1) -> np.ndarray:
    """Boolean mask of elements outside the 1-ulp rule (NaN must match NaN)."""
    got, want = np.asarray(got), np.asarray(want)
    gn, wn = bf16_isnan(got), bf16_isnan(want)
    far = np.abs(bf16_key(got) - bf16_key(want)) > max_ulp
    return np.where(gn | wn, gn != wn, far)


def bf16_interval_violations(got, lo, hi) -> np.ndarray:
    got = np.asarray(got)
    gn, ln, hn = bf16_isnan(got), bf16_isnan(lo), bf16_isnan(hi)
    k = bf16_key(got)
    out = (k < bf16_key(lo)) | (k > bf16_key(hi))
    return np.where(gn | ln | hn, ~(gn & (ln | hn)), out)


def rel_violations(got, want, rtol: float, floor=None) -> np.ndarray:
    """|got - want| > rtol * max(|want|, floor) (floor broadcastable); NaN/inf must match."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    scale = np.abs(want) if floor is None else np.maximum(np.abs(want), floor)
    fin = np.isfinite(got) & np.isfinite(want)
    bad = np.abs(got - want) > rtol * scale
    same_special = (np.isnan(got) & np.isnan(want)) | (np.isinf(got) & np.isinf(want) & (np.sign(got) == np.sign(want)))
    return np.where(fin, bad, ~same_special)
