"""Seeded synthetic inputs for the row-normalisation path.

This module only draws numbers: it holds none of the method's arithmetic and
is shared by the tests (CUDA path and oracle alike) and by the benchmark.
Every draw is made on the host in float32 from ``numpy.random.Generator``
(PCG64) in a fixed tensor order; bf16 tensors are float32 draws rounded to
nearest-even by torch's CPU conversion and carried as their uint16 bit
patterns, so every consumer reads identical bits.

Shapes follow the sources:
  * weight rows: the DragonScale package description ("Kernels and speed":
    an 11008 x 4096 weight; "Measured": 768 -> 2048 layers) and the tern-tc
    decoder's "100m" size (12 layers, d_model 768, 12 query / 4 kv heads of
    64, d_ff 2048, vocab 32000, tied embedding);
  * activation rows: TensorFold PR #1260 (Dory widths 4,096 and 7,168, rows to
    8,192 and beyond).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class WeightSeg:
    """One weight matrix: fp32 rows, per-row gain, upstream gradient."""

    name: str
    w: np.ndarray                 # float32 [rows, cols]
    g: np.ndarray | None          # float32 [rows] or None (mode "unit")
    gy: np.ndarray                # float32 or bf16 bits (uint16) [rows, cols]
    radius: float = 1.0

    @property
    def rows(self) -> int:
        return self.w.shape[0]

    @property
    def cols(self) -> int:
        return self.w.shape[1]


@dataclass
class ActRows:
    """Activation rows: bf16 x (slerp: res), optional bf16 r (slerp: out), fp32 alpha."""

    name: str
    x: np.ndarray                 # uint16 [rows, cols]
    r: np.ndarray | None          # uint16 [rows, cols]
    alpha: np.ndarray | None = None  # float32 [cols]

    @property
    def rows(self) -> int:
        return self.x.shape[0]

    @property
    def cols(self) -> int:
        return self.x.shape[1]


@dataclass
class Workload:
    name: str
    eps: float
    weights: list[WeightSeg] = field(default_factory=list)
    acts: list[ActRows] = field(default_factory=list)
    weff_dtype: str = "bf16"      # "bf16" | "f32"
    gy_dtype: str = "bf16"


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def drifted_rows(rng, rows: int, cols: int, std: float) -> np.ndarray:
    """N(0, std) entries times a per-row lognormal(0, 1) factor (row drift)."""
    w = rng.standard_normal((rows, cols), dtype=np.float32)
    w *= np.float32(std)
    w *= np.exp(rng.standard_normal((rows, 1), dtype=np.float32))
    return w


def gains(rng, rows: int) -> np.ndarray:
    return rng.uniform(0.5, 2.0, rows).astype(np.float32)


def normal_bf16(rng, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16_bits(a)


def spiked_bf16(rng, rows: int, cols: int, frac: float = 0.01, scale: float = 1e3) -> np.ndarray:
    """N(0,1) rows, round(frac*rows) of them (seeded permutation) times scale, then bf16."""
    a = rng.standard_normal((rows, cols), dtype=np.float32)
    k = int(round(frac * rows))
    idx = rng.permutation(rows)[:k]
    a[idx] *= np.float32(scale)
    return to_bf16_bits(a)


def alpha_vec(rng, cols: int, std: float = 0.05) -> np.ndarray:
    return rng.normal(0.0, std, cols).astype(np.float32)


# ---------------------------------------------------------------------------
# Named workloads.  Draw order is fixed per workload (documented inline).

def tiny(seed: int = 0) -> Workload:
    """W [64,128] N(0,1)*exp(N(0,1)) per row, g U(0.5,2), GY fp32 N(0,1),
    X, R bf16 [32,128] N(0,1), alpha [128] N(0,0.05), eps 1e-6.
    Order: W, row factors, g, GY, X, R, alpha."""
    rng = _rng(seed)
    w = drifted_rows(rng, 64, 128, 1.0)
    g = gains(rng, 64)
    gy = rng.standard_normal((64, 128), dtype=np.float32)
    x = normal_bf16(rng, (32, 128))
    r = normal_bf16(rng, (32, 128))
    a = alpha_vec(rng, 128)
    return Workload("tiny", 1e-6, [WeightSeg("w", w, g, gy)], [ActRows("x", x, r, a)],
                    weff_dtype="f32", gy_dtype="f32")


def mlp_pair(seed: int = 0) -> Workload:
    """up [2048,768], down [768,2048] fp32 N(0,0.02)*lognormal rows, g U(0.5,2),
    GY bf16 N(0,1e-3); bf16 W_eff.  Order per matrix: W, factors, g, GY."""
    rng = _rng(seed)
    segs = []
    for name, (R, C) in (("up", (2048, 768)), ("down", (768, 2048))):
        w = drifted_rows(rng, R, C, 0.02)
        g = gains(rng, R)
        gy = normal_bf16(rng, (R, C), 1e-3)
        segs.append(WeightSeg(name, w, g, gy))
    return Workload("mlp_pair", 1e-6, segs)


def activations(seed: int = 0, rows: int = 16384, cols: int = 4096) -> Workload:
    """X, R bf16 [rows, cols] N(0,1) with 1% of rows (each tensor its own
    permutation) times 1e3; alpha [cols] N(0,0.05); eps 1e-6.
    Order: X (values, permutation), R (values, permutation), alpha."""
    rng = _rng(seed)
    x = spiked_bf16(rng, rows, cols)
    r = spiked_bf16(rng, rows, cols)
    a = alpha_vec(rng, cols)
    return Workload(f"activations_{rows}x{cols}", 1e-6, [], [ActRows("x", x, r, a)])


LAYER_SHAPES = (("q", 768, 768), ("k", 256, 768), ("v", 256, 768), ("o", 768, 768),
                ("gate", 2048, 768), ("up", 2048, 768), ("down", 768, 2048))


def whole_model(seed: int = 0, n_layer: int = 12, vocab: int = 32000) -> Workload:
    """Every weight of a 12-layer d_model 768 decoder (GQA 12/4 heads of 64,
    SwiGLU d_ff 2048) plus the tied embedding [vocab, 768]: 85 segments.
    fp32 N(0,0.02)*lognormal rows, g U(0.5,2), GY bf16 N(0,1e-3).
    Order: layer 0..11 in LAYER_SHAPES order, then the embedding; per
    segment W, factors, g, GY."""
    rng = _rng(seed)
    segs = []
    for layer in range(n_layer):
        for name, R, C in LAYER_SHAPES:
            w = drifted_rows(rng, R, C, 0.02)
            segs.append(WeightSeg(f"l{layer}.{name}", w, gains(rng, R), normal_bf16(rng, (R, C), 1e-3)))
    w = drifted_rows(rng, vocab, 768, 0.02)
    segs.append(WeightSeg("embed", w, gains(rng, vocab), normal_bf16(rng, (vocab, 768), 1e-3)))
    return Workload("whole_model", 1e-6, segs)


def wide(seed: int = 0) -> Workload:
    """Weights [14336,4096] and [4096,14336] fp32 with gains, bf16 GY;
    activations [8192,7168] and [4096,16384] N(0,1) with alpha.
    Order: weight 1 (W, factors, g, GY), weight 2, act 1 (X, R, alpha), act 2."""
    rng = _rng(seed)
    segs = []
    for name, (R, C) in (("w_14336x4096", (14336, 4096)), ("w_4096x14336", (4096, 14336))):
        w = drifted_rows(rng, R, C, 0.02)
        segs.append(WeightSeg(name, w, gains(rng, R), normal_bf16(rng, (R, C), 1e-3)))
    acts = []
    for name, (R, C) in (("x_8192x7168", (8192, 7168)), ("x_4096x16384", (4096, 16384))):
        acts.append(ActRows(name, normal_bf16(rng, (R, C)), normal_bf16(rng, (R, C)), alpha_vec(rng, C)))
    return Workload("wide", 1e-6, segs, acts)


def long_rows(seed: int = 0, w_rows: int = 6, w_cols: int = 262144,
              a_rows: int = 4, a_cols: int = 262144) -> Workload:
    """Rows past the single-pass limit (more than 8 CTAs' staged slices):
    fp32 weights [6, 262144] with gains and bf16 GY, bf16 activations
    [4, 262144] with alpha."""
    rng = _rng(seed)
    w = drifted_rows(rng, w_rows, w_cols, 0.02)
    seg = WeightSeg("w_long", w, gains(rng, w_rows), normal_bf16(rng, (w_rows, w_cols), 1e-3))
    act = ActRows("x_long", normal_bf16(rng, (a_rows, a_cols)), normal_bf16(rng, (a_rows, a_cols)),
                  alpha_vec(rng, a_cols))
    return Workload("long_rows", 1e-6, [seg], [act])


def with_fp32_state(weights: list[WeightSeg], seed: int, std: float = 1e-3) -> list[WeightSeg]:
    """The same weight rows, each paired with an fp32 [rows, cols] N(0, std)
    tensor in `gy`: the gradient G (before the optimizer step) or the
    momentum m (after it) of method "rescale".  Drawn in segment order."""
    rng = _rng(seed)
    return [WeightSeg(s.name, s.w, s.g, (rng.standard_normal(s.w.shape, dtype=np.float32) * np.float32(std)),
                      s.radius) for s in weights]


def small_norm_rows(seed: int, rows: int, cols: int, sumsq: float = 1e-5) -> np.ndarray:
    """bf16 rows with sum of squares near `sumsq` (eps-sensitive control set)."""
    rng = _rng(seed)
    a = rng.standard_normal((rows, cols), dtype=np.float32)
    a *= np.float32(np.sqrt(sumsq / cols))
    return to_bf16_bits(a)


def integer_rows(seed: int, rows: int, cols: int, max_sumsq: int = (1 << 24) - 1) -> np.ndarray:
    """bf16 rows of small integers whose sum of squares stays below max_sumsq
    (exact in fp32) yet far above fp16's largest finite value."""
    rng = _rng(seed)
    lim = int(np.floor(np.sqrt(max_sumsq / cols)))
    lim = max(1, min(lim, 256))           # |v| <= 256 is exact in bf16
    a = rng.integers(-lim, lim + 1, size=(rows, cols)).astype(np.float32)
    return to_bf16_bits(a)


@dataclass
class QKRows:
    """Dory's attention rows for tf_qk_rows_l2: q [R, hq*D], k and v [R, hk*D]
    bf16 bits, positions [R] int32, inverse frequencies fp32 [D/2], q's scale
    vector fp32 [hq*D]."""

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    pos: np.ndarray
    inv: np.ndarray
    q_scale: np.ndarray
    head_dim: int
    hq: int
    hk: int

    @property
    def rows(self) -> int:
        return self.q.shape[0]


def rope_inv(head_dim: int, theta: float = 10000.0) -> np.ndarray:
    """1 / theta^(2i/D) in fp32 steps, the way the tern-tc listing forms its
    RoPE cache (rope_cache): the exponent, the power and the reciprocal each
    rounded to fp32."""
    e = np.arange(0, head_dim, 2, dtype=np.float32) / np.float32(head_dim)
    return (np.float32(1.0) / np.power(np.float32(theta), e, dtype=np.float32)).astype(np.float32)


def qk_rows(seed: int = 0, rows: int = 2048, head_dim: int = 256, hq: int = 16, hk: int = 4,
            theta: float = 10000.0, far_pos: int = 199_800) -> QKRows:
    """q, k, v ~ N(0,1) bf16; the first two thirds of the rows at positions
    0, 1, ... and the last third at far_pos, far_pos + 1, ...; q_scale ~
    U(0.5, 2) fp32 (the pages form it on the host and give no values)."""
    rng = _rng(seed)
    q = normal_bf16(rng, (rows, hq * head_dim))
    k = normal_bf16(rng, (rows, hk * head_dim))
    v = normal_bf16(rng, (rows, hk * head_dim))
    near = rows - rows // 3
    pos = np.concatenate([np.arange(near), far_pos + np.arange(rows - near)]).astype(np.int32)
    q_scale = rng.uniform(0.5, 2.0, hq * head_dim).astype(np.float32)
    return QKRows(q, k, v, pos, rope_inv(head_dim, theta), q_scale, head_dim, hq, hk)
