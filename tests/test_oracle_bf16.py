"""Pins for the oracle's f64 -> bf16 rounding (round to nearest, ties to even).

Checked against (a) a brute-force nearest search over every finite bf16
value with exact rational arithmetic, and (b) torch's float32 -> bfloat16
conversion for values float32 can hold.  Neither shares code with the oracle.
"""
from __future__ import annotations

import bisect
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _bits_value(b: int) -> Fraction:
    e, m = (b >> 7) & 0xFF, b & 0x7F
    v = Fraction(m) * Fraction(2) ** -133 if e == 0 else Fraction(128 + m) * Fraction(2) ** (e - 134)
    return -v if b & 0x8000 else v


# every non-negative finite bf16, sorted by value (bits 0x0000..0x7F7F are monotone)
_POS = list(range(0x0000, 0x7F80))
_POS_VAL = [_bits_value(b) for b in _POS]
_OVERFLOW = _POS_VAL[-1] + (_POS_VAL[-1] - _POS_VAL[-2]) / 2  # max + half its quantum


def brute_rne(v: float) -> int:
    if math.isnan(v):
        return 0x7FC0 | (0x8000 if math.copysign(1, v) < 0 else 0)
    sign = 0x8000 if math.copysign(1.0, v) < 0 else 0
    a = Fraction(abs(v)) if math.isfinite(v) else None
    if a is None or a >= _OVERFLOW:
        return sign | 0x7F80
    i = bisect.bisect_left(_POS_VAL, a)
    if i < len(_POS_VAL) and _POS_VAL[i] == a:
        return sign | _POS[i]
    lo, hi = i - 1, i
    dlo, dhi = a - _POS_VAL[lo], _POS_VAL[hi] - a
    if dlo < dhi or (dlo == dhi and _POS[lo] % 2 == 0):
        return sign | _POS[lo]
    return sign | _POS[hi]


def _samples(n: int, seed: int) -> list[float]:
    rng = np.random.default_rng(seed)
    out = []
    # log-uniform magnitudes over and beyond bf16's range, both signs
    exps = rng.uniform(-160, 140, n)
    mant = rng.uniform(1.0, 2.0, n)
    sgn = rng.choice([-1.0, 1.0], n)
    out += list(sgn * mant * np.exp2(np.floor(exps)))
    return out


def _ties() -> list[float]:
    """Values exactly halfway between neighbouring bf16 values (both parities)."""
    out = []
    for b in (0x0001, 0x0002, 0x007F, 0x0080, 0x0081, 0x3F80, 0x3F81, 0x3F1A, 0x4000, 0x7F7E):
        v0, v1 = _bits_value(b), _bits_value(b + 1)
        mid = (v0 + v1) / 2
        out.append(float(mid))  # exact: 9 significant bits
        out.append(-float(mid))
    return out


def test_rne_against_brute_force():
    vals = _samples(4000, 1) + _ties() + [0.0, -0.0, 1.0, -1.0, 0.6, 0.8, 1e-45, 2.0 ** -133, 2.0 ** -134,
                                          3 * 2.0 ** -135, 2.0 ** -126, 3.3895313892515355e38,
                                          3.3961775292304957e38, 3.4e38, 1e300, -1e300, 5e-324]
    bad = [(v, oracle.bf16_rne(v), brute_rne(v)) for v in vals if oracle.bf16_rne(v) != brute_rne(v)]
    assert not bad, bad[:5]


def test_overflow_boundary():
    top = float(_OVERFLOW)  # exactly (2 - 2^-8) * 2^127: a tie that rounds to 2^128 -> inf
    assert oracle.bf16_rne(top) == 0x7F80
    assert oracle.bf16_rne(math.nextafter(top, 0)) == 0x7F7F
    assert oracle.bf16_rne(-top) == 0xFF80


def test_specials():
    assert oracle.bf16_rne(float("inf")) == 0x7F80
    assert oracle.bf16_rne(float("-inf")) == 0xFF80
    assert oracle.bf16_rne(0.0) == 0x0000
    assert oracle.bf16_rne(-0.0) == 0x8000
    assert (oracle.bf16_rne(float("nan")) & 0x7F80) == 0x7F80 and (oracle.bf16_rne(float("nan")) & 0x7F)
    # the smallest subnormal's halfway point ties to even (zero)
    assert oracle.bf16_rne(2.0 ** -134) == 0x0000
    assert oracle.bf16_rne(math.nextafter(2.0 ** -134, 1)) == 0x0001


def test_value_roundtrip_all_patterns():
    for b in range(0x10000):
        v = oracle.bf16_value(b)
        e = (b >> 7) & 0xFF
        if e == 0xFF and (b & 0x7F):
            assert math.isnan(v)
            continue
        assert oracle.bf16_rne(v) == b
        if e != 0xFF:
            assert Fraction(v) == _bits_value(b)


def test_matches_torch_for_float32_values():
    rng = np.random.default_rng(7)
    f = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(20000) * np.exp2(rng.integers(-140, 120, 20000))).astype(np.float32),
        np.array([np.finfo(np.float32).max, np.finfo(np.float32).tiny, 1e-45, -1e-45], np.float32),
    ])
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("v,bits", [(0.6, 0x3F1A), (0.8, 0x3F4D), (1.0, 0x3F80), (0.5, 0x3F00),
                                    (2.0 / 3.0, 0x3F2B), (2 ** -0.5, 0x3F35)])
def test_hand_values(v, bits):
    assert oracle.bf16_rne(v) == bits


def test_array_rounding_matches_scalar():
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.standard_normal(3000) * np.exp2(rng.integers(-140, 130, 3000)),
                        [0.0, -0.0, np.inf, -np.inf, 1e300]])
    arr = oracle.bf16_rne_array(v)
    assert [int(b) for b in arr] == [oracle.bf16_rne(float(x)) for x in v]
