#!/usr/bin/env python
"""Benchmark of the per-row L2 normalisation hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:

  1. ds_wn_forward   every weight of a 12-layer d_model-768 decoder plus its
                     tied embedding (85 segments, 114,944 rows, 100,073,472
                     fp32 elements) -> bf16 W_eff, one call
  2. ds_l2_rows      activation rows X [16384, 4096] bf16
  3. ds_wn_backward  the same 85 segments, bf16 GY -> fp32 grad_w, grad_g
  4. ds_l2_rows      X + R (fused residual add)
  5. ds_row_renorm   the 85 segments in place
  6. ds_slerp_rows   res = X, out = R, alpha [4096]

Every call reads more than the 126 MB L2 and consecutive calls touch
disjoint buffers (>= 268 MB of other traffic between two uses of one
buffer), so inputs come from HBM without an explicit flush.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config step|mlp_pair|wide|optimizer|act_backward|dory|gain|long_rows]
                    [--no-extras]

`--config` selects another workload for a per-call report (default: the
step above); after the default step, every other workload's calls are
timed and reported under "extras" (skip with --no-extras).  mlp_pair = up [2048,768] + down [768,2048] (fwd, bwd, renorm;
L2-resident, so each timed step uses the next of 16 buffer copies and a
CUDA-graph replay of the calls is timed as well).  wide = weights
[14336,4096], [4096,14336] (fwd, bwd) and activation rows [8192,7168],
[4096,16384] (l2, l2 + residual, slerp).  optimizer = ds_grad_project and
ds_renorm_momentum over the whole-model weights.  act_backward = the
backward of the activation calls on [16384,4096] (upstream gradient bf16).
dory = Dory's gated and SwiGLU l2 rows on [16384,4096] and [8192,7168]
(scale vectors fp32 U(0.5, 2)) and its q/k rows on 16384 rows of 16 + 4 + 4
heads of 256.  gain = the row lengths and the scalar-gain backward of the
whole model, and forward + backward of 12 GPT-2 XL Conv1D weights
[1600, 6400] stored [in, out] (transposed rows).  long_rows = rows split
over a cluster ([2048,40000] forward, [4096,24576] slerp) and rows on the
two-pass stream ([256,262144] forward, [512,262144] slerp).

Prints one JSON line (rank 0).  `value` is algorithmic bytes moved by all
ranks per second (GB/s); per-kernel GB/s and rows/s, the roofline of the
dominant kernel, the end-to-end figure through the C ABI from pinned host
buffers, and the float64 CPU oracle timed on a bounded sample ride along.
Under torchrun every rank runs the same step on its own seeded data (weak
scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes as ct
import hashlib
import json
import os
import statistics
import sys
import threading
import time
import types

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "achieved HBM GB/s (fraction of B200 peak) and rows/s per kernel, fwd+bwd"
EPS = 1e-6
ACT_ROWS, ACT_COLS = 16384, 4096
QK_ROWS = 16384
WORKLOAD = ("whole-model weights: 85 segments (12 layers x {q,k,v,o,gate,up,down} + tied embedding "
            "[32000,768]), 100,073,472 fp32 elements, fwd (bf16 W_eff) + bwd (bf16 GY) + renorm; "
            "activation rows [16384,4096] bf16: l2, l2 + residual, slerp")
WORKLOADS = {
    "step": WORKLOAD,
    "mlp_pair": "MLP pair: up [2048,768] + down [768,2048] fp32 rows, one segment table, fwd (bf16 W_eff) + "
                "bwd (bf16 GY) + renorm; 16 rotating buffer copies",
    "wide": "wide rows: weights [14336,4096] and [4096,14336] fp32 (fwd bf16 W_eff, bwd bf16 GY), activation "
            "rows [8192,7168] and [4096,16384] bf16 (l2, l2 + residual, slerp)",
    "optimizer": "optimizer companions of method rescale on the whole-model weights (85 segments, 100,073,472 "
                 "fp32 elements): gradient projection before the step, momentum projection + renorm after it "
                 "(fp32 gradient and momentum, in place)",
    "act_backward": "activation backward on rows [16384,4096] bf16: l2 (dx fp32), l2 with residual, slerp "
                    "(dres, dout fp32 and dalpha [4096] through its workspace)",
    "gain": "row lengths (Monitor) and the scalar-gain backward (bf16 GY) of the whole-model weights (85 "
            "segments, 100,073,472 fp32 elements); forward (bf16 W_eff) and backward (bf16 GY) of 12 GPT-2 XL "
            "Conv1D weights [1600, 6400] stored [in, out] (transposed rows, 122,880,000 elements)",
    "long_rows": "rows longer than one CTA's shared memory: wn_forward [2048,40000] and slerp_rows [4096,24576] "
                 "(clusters of 4 and 2 CTAs, each staging a slice of the row; partial sums through distributed "
                 "shared memory), wn_forward [256,262144] and slerp_rows [512,262144] (the two-pass stream); inputs "
                 "drawn on the device",
    "dory": "Dory's fused activation rows: gated l2 rows (o, g bf16, sg fp32) and SwiGLU l2 rows (g, u bf16, "
            "sug, suu fp32) on [16384,4096] and [8192,7168]; q/k rows (rotate-half RoPE, per-head l2, q scale; "
            "16 q heads over 4 kv heads of 256, v copied to the cache) on 16384 rows, a third past position 199,800",
}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the per-call report of the other workloads after the default step")
    p.add_argument("--config", choices=tuple(WORKLOADS), default="step")
    return p.parse_args()


# ------------------------------------------------------------ bookkeeping --

def call_bytes(kind: str, segs=None, act=None) -> int:
    """Algorithmic bytes of one call: every input read once, every output
    written once (per-row gains and grad_g 4 B per row)."""
    if kind == "qk":   # q read + written, k and v read + written to the cache, pos; inv and q_scale per call
        wq, wk = act.hq * act.head_dim * 2, act.hk * act.head_dim * 2
        return act.rows * (2 * wq + 4 * wk + 4) + act.head_dim // 2 * 4 + act.hq * act.head_dim * 4
    if act is not None:
        A = act.rows * act.cols
        return {"l2": A * (2 + 2), "l2res": A * (2 + 2 + 2), "slerp": A * (2 + 2 + 2) + act.cols * 4,
                "l2bwd": A * (2 + 2 + 4), "l2resbwd": A * (2 + 2 + 2 + 4),
                "slerpbwd": A * (2 + 2 + 2 + 4 + 4) + act.cols * (4 + 4),
                "gate": A * (2 + 2 + 2) + act.cols * 4, "swiglu": A * (2 + 2 + 2) + act.cols * (4 + 4)}[kind]
    E = sum(s.w.size for s in segs)
    R = sum(unit_rows(s) for s in segs)
    return {"fwd": E * (4 + 2) + R * 4, "bwd": E * (4 + 2 + 4) + R * (4 + 4), "renorm": E * (4 + 4),
            "project": E * (4 + 4 + 4), "momentum": E * (4 + 4 + 4 + 4), "norms": E * 4 + R * 4,
            # scalar gain: grad_w, the per-row parts, then their sum re-reads the parts
            "bwd_scalar": E * (4 + 2 + 4) + R * (4 + 4) + len(segs) * 8}[kind]


def unit_rows(s) -> int:
    """Unit rows of a weight segment: its rows, or for a transposed
    (Conv1D, stored [in, out]) segment its stored columns."""
    return s.w.shape[1] if getattr(s, "transposed", False) else s.w.shape[0]


def call_rows(kind: str, segs=None, act=None) -> int:
    return act.rows if act is not None else sum(unit_rows(s) for s in segs)


def step_bytes(weights, act_rows=ACT_ROWS, act_cols=ACT_COLS) -> dict[str, int]:
    """Bytes of the six calls of the default step for these weights and
    activation-row shape."""
    act = types.SimpleNamespace(rows=act_rows, cols=act_cols)
    return {"wn_forward": call_bytes("fwd", weights), "l2_rows": call_bytes("l2", act=act),
            "wn_backward": call_bytes("bwd", weights), "l2_rows_residual": call_bytes("l2res", act=act),
            "row_renorm": call_bytes("renorm", weights), "slerp_rows": call_bytes("slerp", act=act)}


def plan(config: str, seed: int):
    """(weight groups, activation groups, calls, buffer copies) of a workload.
    A call is (name, kind, group); kinds fwd/bwd/renorm take a weight group
    (a segment table), l2/l2res/slerp an activation group."""
    from l2_row_b200 import workloads as wl

    if config == "step":
        wg = {"model": wl.whole_model(seed).weights}
        ag = {"x": wl.activations(seed, ACT_ROWS, ACT_COLS).acts[0]}
        calls = [("wn_forward", "fwd", "model"), ("l2_rows", "l2", "x"), ("wn_backward", "bwd", "model"),
                 ("l2_rows_residual", "l2res", "x"), ("row_renorm", "renorm", "model"), ("slerp_rows", "slerp", "x")]
        return wg, ag, calls, 1
    if config == "mlp_pair":
        wg = {"mlp": wl.mlp_pair(seed).weights}
        calls = [("wn_forward", "fwd", "mlp"), ("wn_backward", "bwd", "mlp"), ("row_renorm", "renorm", "mlp")]
        return wg, {}, calls, 16
    if config == "wide":
        w = wl.wide(seed)
        wg = {s.name[2:]: [s] for s in w.weights}
        ag = {a.name[2:]: a for a in w.acts}
        calls = []
        for g in wg:
            calls += [(f"wn_forward_{g}", "fwd", g), (f"wn_backward_{g}", "bwd", g)]
        for g in ag:
            calls += [(f"l2_rows_{g}", "l2", g), (f"l2_rows_residual_{g}", "l2res", g), (f"slerp_rows_{g}", "slerp", g)]
        return wg, ag, calls, 1
    if config == "act_backward":
        ag = {"x": wl.activations(seed, ACT_ROWS, ACT_COLS).acts[0]}
        calls = [("l2_rows_backward", "l2bwd", "x"), ("l2_rows_residual_backward", "l2resbwd", "x"),
                 ("slerp_rows_backward", "slerpbwd", "x")]
        return {}, ag, calls, 1
    if config == "dory":
        ag = {"x": wl.activations(seed, ACT_ROWS, ACT_COLS).acts[0],
              "7168": wl.activations(seed + 1, 8192, 7168).acts[0]}
        calls = []
        for g in ag:
            sfx = "" if g == "x" else f"_{g}"
            calls += [(f"gate_l2_rows{sfx}", "gate", g), (f"swiglu_l2_rows{sfx}", "swiglu", g)]
        ag["qk"] = wl.qk_rows(seed, rows=QK_ROWS)
        calls.append(("qk_rows_l2", "qk", "qk"))
        return {}, ag, calls, 1
    if config == "gain":
        import types as _types

        rng = np.random.default_rng(seed + 21)
        conv = []
        for layer in range(12):   # GPT-2 XL mlp c_fc: Conv1D(nf=6400, nx=1600) keeps weight [1600, 6400]
            w = np.ascontiguousarray(wl.drifted_rows(rng, 6400, 1600, 0.02).T)
            conv.append(_types.SimpleNamespace(name=f"c_fc{layer}", w=w, g=wl.gains(rng, 6400),
                                               gy=wl.normal_bf16(rng, (1600, 6400), 1e-3), radius=1.0,
                                               transposed=True, rows=1600, cols=6400))
        wg = {"model": wl.whole_model(seed).weights, "conv1d": conv}
        calls = [("row_norms", "norms", "model"), ("wn_backward_scalar_gain", "bwd_scalar", "model"),
                 ("wn_forward_conv1d", "fwd", "conv1d"), ("wn_backward_conv1d", "bwd", "conv1d")]
        return wg, {}, calls, 1
    if config == "optimizer":
        wg = {"model": wl.with_fp32_state(wl.whole_model(seed).weights, seed + 1)}
        calls = [("grad_project", "project", "model"), ("renorm_momentum", "momentum", "model")]
        return wg, {}, calls, 1
    raise ValueError(config)


def max_over_ranks(dist, values: list[float], device) -> list[float]:
    """Element-wise maximum of per-rank timings (ms).  Every rank calls it at
    the same point with the same number of values; without a process group
    the values come back unchanged."""
    if dist is None:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_gbs(world: int, bytes_per_rank: int, ms_per_step: float) -> float:
    """Aggregate GB/s over all ranks: each rank processes its own copy of the
    step's bytes (weak scaling) in at most the slowest rank's time."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


def measured_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_digest() -> str:
    """Digest of the sources of the default step's kernels (every call of the
    step runs k_tile) and of the host code that plans their launches."""
    h = hashlib.sha256()
    for rel in ("l2_row_b200/csrc/ds_tile.cu", "l2_row_b200/csrc/ds_api.cpp",
                "l2_row_b200/csrc/ds_device.cuh", "l2_row_b200/csrc/ds_internal.h"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec["kernels"][kernel]
        if rec.get("source_digest") != kernel_source_digest():
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
                rs = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._ok:
            self._t.join()
        return False

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ------------------------------------------------------------- our arm -----

class Step:
    """Device buffers, prebuilt C segment tables and the calls of one step of
    a workload (see `plan`), in `copies` independent buffer sets."""

    def __init__(self, seed: int, config: str = "step"):
        import torch

        from l2_row_b200 import ds
        from l2_row_b200 import workloads as wl

        self.torch, self.ds = torch, ds
        self.wg, self.ag, self.plan, self.copies = plan(config, seed)
        dev = "cuda"

        def f32(a):
            return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)

        def bf16(b):
            return torch.from_numpy(np.ascontiguousarray(b, np.uint16).view(np.int16)).to(dev).view(torch.bfloat16)

        # per weight group: one flat buffer per tensor kind the plan uses
        # (few, large H2D copies in the e2e leg)
        self.wbuf, self.abuf = {}, {}
        self.inputs, self.outputs = [], []   # (device tensor, host array) / device tensors of copy 0
        for name, segs in self.wg.items():
            kinds = {k for _, k, g in self.plan if g == name}
            state = bool(kinds & {"project", "momentum"})   # gy holds the fp32 gradient / momentum
            host = {"w": np.concatenate([s.w.ravel() for s in segs]),
                    "gy": np.concatenate([s.gy.ravel() for s in segs]),
                    "gain": np.concatenate([s.g for s in segs])}
            n_el, n_rows = host["w"].size, host["gain"].size
            copies = []
            for c in range(self.copies):
                b = {"w": f32(host["w"])}
                if kinds & {"fwd", "bwd"}:
                    b["gain"] = f32(host["gain"])
                if "fwd" in kinds:
                    b["weff"] = torch.empty(n_el, dtype=torch.bfloat16, device=dev)
                if kinds & {"bwd", "bwd_scalar"}:
                    b["gy"] = bf16(host["gy"])
                    b["grad_w"] = torch.empty(n_el, dtype=torch.float32, device=dev)
                    b["grad_g"] = torch.empty(n_rows + len(segs), dtype=torch.float32, device=dev)
                if "bwd_scalar" in kinds:   # one gain per segment
                    b["gscalar"] = torch.full((len(segs),), 0.5, dtype=torch.float32, device=dev)
                if "norms" in kinds:
                    b["rnorm"] = torch.empty(n_rows, dtype=torch.float32, device=dev)
                if state:
                    b["state"] = f32(host["gy"])
                copies.append(b)
            self.wbuf[name] = copies
            b0 = copies[0]
            self.inputs.append((b0["w"], host["w"]))
            if "gain" in b0:
                self.inputs.append((b0["gain"], host["gain"]))
            if "gy" in b0:
                self.inputs.append((b0["gy"], host["gy"].view(np.int16)))
            if "state" in b0:
                self.inputs.append((b0["state"], host["gy"]))
            if "gscalar" in b0:
                self.inputs.append((b0["gscalar"], np.full(len(segs), 0.5, np.float32)))
            self.outputs += [b0[k] for k in ("weff", "grad_w", "grad_g", "state", "rnorm") if k in b0]
            if kinds & {"renorm", "momentum"}:
                self.outputs.append(b0["w"])
        for name, a in self.ag.items():
            kinds = {k for _, k, g in self.plan if g == name}
            if kinds == {"qk"}:
                def i32(x):
                    return torch.from_numpy(np.ascontiguousarray(x, np.int32)).to(dev)

                copies = []
                for c in range(self.copies):
                    b = {"q": bf16(a.q), "k": bf16(a.k), "v": bf16(a.v), "pos": i32(a.pos), "inv": f32(a.inv),
                         "q_scale": f32(a.q_scale)}
                    b.update({"q_out": torch.empty_like(b["q"]), "k_cache": torch.empty_like(b["k"]),
                              "v_cache": torch.empty_like(b["v"])})
                    copies.append(b)
                self.abuf[name] = copies
                b0 = copies[0]
                self.inputs += [(b0["q"], a.q.view(np.int16)), (b0["k"], a.k.view(np.int16)),
                                (b0["v"], a.v.view(np.int16)), (b0["pos"], a.pos), (b0["inv"], a.inv),
                                (b0["q_scale"], a.q_scale)]
                self.outputs += [b0["q_out"], b0["k_cache"], b0["v_cache"]]
                continue
            bwd = any(k.endswith("bwd") for k in kinds)
            dy_host = scales = None
            if kinds & {"gate", "swiglu"}:   # per-column scales U(0.5, 2), seeded after the rows
                srng = np.random.default_rng(seed + 11)
                scales = [srng.uniform(0.5, 2.0, a.cols).astype(np.float32) for _ in range(2)]
            if bwd:   # the upstream gradient: bf16 N(0,1), seeded after the rows
                dy_host = wl.normal_bf16(np.random.default_rng(seed + 7), a.x.shape)
            copies = []
            for c in range(self.copies):
                x = bf16(a.x)
                b = {"x": x, "r": bf16(a.r), "alpha": f32(a.alpha)}
                if scales is not None:
                    b["sa"], b["sb"] = f32(scales[0]), f32(scales[1])
                if bwd:
                    b["dy"] = bf16(dy_host)
                    b["dx"] = torch.empty(a.x.shape, dtype=torch.float32, device=dev)
                    b["dx2"] = torch.empty_like(b["dx"])
                    b["dres"] = torch.empty_like(b["dx"])
                    b["dout"] = torch.empty_like(b["dx"])
                    b["dalpha"] = torch.empty(a.cols, dtype=torch.float32, device=dev)
                    b["ws"] = torch.empty(ds.ds_slerp_rows_backward_workspace(a.cols), dtype=torch.uint8, device=dev)
                else:
                    b.update({"y": torch.empty_like(x), "y2": torch.empty_like(x), "h": torch.empty_like(x)})
                copies.append(b)
            self.abuf[name] = copies
            b0 = copies[0]
            self.inputs += [(b0["x"], a.x.view(np.int16)), (b0["r"], a.r.view(np.int16)), (b0["alpha"], a.alpha)]
            if scales is not None:
                self.inputs += [(b0["sa"], scales[0]), (b0["sb"], scales[1])]
            if bwd:
                self.inputs.append((b0["dy"], dy_host.view(np.int16)))
                self.outputs += [b0["dx"], b0["dx2"], b0["dres"], b0["dout"], b0["dalpha"]]
            else:
                self.outputs += [b0["y"], b0["y2"], b0["h"]]

        self.names = [c[0] for c in self.plan]
        self.bytes = {}
        self.rows = {}
        for name, kind, g in self.plan:
            segs, act = (self.wg[g], None) if g in self.wg else (None, self.ag[g])
            self.bytes[name] = call_bytes(kind, segs, act)
            self.rows[name] = call_rows(kind, segs, act)

        lib = ds.lib()
        eps = ct.c_float(EPS)
        self.tables = []
        self.calls = []   # [copy][call] -> fn(stream)
        for c in range(self.copies):
            fns = []
            for name, kind, g in self.plan:
                if g in self.wg:
                    b, segs = self.wbuf[g][c], self.wg[g]
                    rows = []
                    eo = ro = 0
                    for si, sgm in enumerate(segs):
                        R, C = sgm.w.shape          # as stored
                        tr = bool(getattr(sgm, "transposed", False))
                        U = unit_rows(sgm)
                        sl = slice(eo, eo + R * C)
                        w = b["w"][sl].view(R, C)
                        gain = b["gain"][ro:ro + U] if "gain" in b else None
                        if kind == "fwd":
                            rows.append(ds.WSeg(w=w, gain=gain, w_eff=b["weff"][sl].view(R, C), transposed=tr).to_c())
                        elif kind == "bwd":
                            rows.append(ds.WSeg(w=w, gain=gain, gy=b["gy"][sl].view(R, C),
                                                grad_w=b["grad_w"][sl].view(R, C),
                                                grad_g=b["grad_g"][ro:ro + U], transposed=tr).to_c())
                        elif kind == "bwd_scalar":   # grad_g: the parts then their sum, U + 1 per segment
                            rows.append(ds.WSeg(w=w, gain=b["gscalar"][si:si + 1], gy=b["gy"][sl].view(R, C),
                                                grad_w=b["grad_w"][sl].view(R, C),
                                                grad_g=b["grad_g"][ro + si:ro + si + U + 1], radius=sgm.radius,
                                                gain_scalar=True).to_c())
                        elif kind == "norms":
                            rows.append(ds.WSeg(w=w, rnorm=b["rnorm"][ro:ro + U]).to_c())
                        elif kind in ("project", "momentum"):
                            rows.append(ds.WSeg(w=w, grad_w=b["state"][sl].view(R, C), radius=sgm.radius).to_c())
                        else:
                            rows.append(ds.WSeg(w=w).to_c())
                        eo += R * C
                        ro += U
                    tab = (ds.ds_wseg * len(rows))(*rows)
                    n = len(rows)
                    fn = {"fwd": lambda s, t=tab, n=n: lib.ds_wn_forward(t, n, ds.DS_BF16, eps, s),
                          "bwd": lambda s, t=tab, n=n: lib.ds_wn_backward(t, n, ds.DS_BF16, eps, s),
                          "bwd_scalar": lambda s, t=tab, n=n: lib.ds_wn_backward(t, n, ds.DS_BF16, eps, s),
                          "norms": lambda s, t=tab, n=n: lib.ds_row_norms(t, n, eps, s),
                          "renorm": lambda s, t=tab, n=n: lib.ds_row_renorm(t, n, eps, s),
                          "project": lambda s, t=tab, n=n: lib.ds_grad_project(t, n, eps, s),
                          "momentum": lambda s, t=tab, n=n: lib.ds_renorm_momentum(t, n, eps, s)}[kind]
                elif kind.endswith("bwd"):
                    b = self.abuf[g][c]
                    if kind == "l2bwd":
                        seg = ds.AGSeg(x=b["x"], dy=b["dy"], dx=b["dx"])
                    elif kind == "l2resbwd":
                        seg = ds.AGSeg(x=b["x"], r=b["r"], dy=b["dy"], dx=b["dx2"])
                    else:
                        seg = ds.AGSeg(x=b["x"], r=b["r"], dy=b["dy"], dx=b["dres"], dr=b["dout"], alpha=b["alpha"])
                    tab = (ds.ds_agseg * 1)(seg.to_c())
                    if kind == "slerpbwd":
                        da, ws = b["dalpha"], b["ws"]
                        fn = (lambda s, t=tab, da=da, ws=ws: lib.ds_slerp_rows_backward(
                            t, 1, eps, da.data_ptr(), ws.data_ptr(), ws.numel(), s))
                    else:
                        fn = lambda s, t=tab: lib.ds_l2_rows_backward(t, 1, eps, s)
                elif kind == "qk":
                    b, a = self.abuf[g][c], self.ag[g]
                    seg = ds.QKSeg(head_dim=a.head_dim, pos=b["pos"], inv_freq=b["inv"], q=b["q"], q_out=b["q_out"],
                                   k=b["k"], k_cache=b["k_cache"], v=b["v"], v_cache=b["v_cache"],
                                   q_scale=b["q_scale"])
                    tab = (ds.ds_qkseg * 1)(seg.to_c())
                    fn = lambda s, t=tab: lib.ds_qk_rows_l2(t, 1, eps, s)
                elif kind in ("gate", "swiglu"):
                    b = self.abuf[g][c]
                    fseg = ds.FSeg(a=b["x"], b=b["r"], y=b["y"], sa=b["sa"], sb=b["sb"] if kind == "swiglu" else None)
                    tab = (ds.ds_fseg * 1)(fseg.to_c())
                    fn = (lambda s, t=tab: lib.ds_gate_l2_rows(t, 1, eps, s)) if kind == "gate" else \
                         (lambda s, t=tab: lib.ds_swiglu_l2_rows(t, 1, eps, s))
                else:
                    b = self.abuf[g][c]
                    if kind == "l2":
                        seg = ds.ASeg(x=b["x"], y=b["y"])
                    elif kind == "l2res":
                        seg = ds.ASeg(x=b["x"], r=b["r"], y=b["y2"])
                    else:
                        seg = ds.ASeg(x=b["x"], r=b["r"], y=b["h"], alpha=b["alpha"])
                    tab = (ds.ds_aseg * 1)(seg.to_c())
                    fn = (lambda s, t=tab: lib.ds_slerp_rows(t, 1, eps, s)) if kind == "slerp" else \
                         (lambda s, t=tab: lib.ds_l2_rows(t, 1, eps, s))
                self.tables.append(tab)
                fns.append(fn)
            self.calls.append(fns)

    def run(self, stream_ptr: int, events=None, k: int = 0) -> None:
        fns = self.calls[k % self.copies]
        for i, name in enumerate(self.names):
            if events is not None:
                events[i].record()
            st = fns[i](stream_ptr)
            if st != 0:
                raise self.ds.DSError(st, name)
        if events is not None:
            events[len(self.names)].record()


# (name, kind, rows, cols): long rows of one length per call, each call's
# inputs larger than L2; drawn on the device from a seeded generator.
LONG_CALLS = [("wn_forward_40000", "fwd", 2048, 40000), ("slerp_rows_24576", "slerp", 4096, 24576),
              ("wn_forward_262144", "fwd", 256, 262144), ("slerp_rows_262144", "slerp", 512, 262144)]


class LongRows:
    """The long-row calls of LONG_CALLS, with the interface of Step that the
    timing loop uses (names, bytes, rows, plan, copies, run).  Weight rows
    are N(0, 0.02) times a per-row lognormal factor with gains U(0.5, 2);
    activation rows bf16 N(0, 1), alpha N(0, 0.05): the recipes of the wide
    workload, drawn on the device (seeded) to keep set-up short."""

    def __init__(self, seed: int):
        import torch

        from l2_row_b200 import ds

        self.torch, self.ds = torch, ds
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1000 + seed)
        lib = ds.lib()
        eps = ct.c_float(EPS)
        self.plan = [(name, kind, None) for name, kind, _, _ in LONG_CALLS]
        self.names = [c[0] for c in self.plan]
        self.copies = 1
        self.bytes, self.rows, self.tables, self.keep, fns = {}, {}, [], [], []
        self.classes = {}
        for name, kind, R, C in LONG_CALLS:
            act = types.SimpleNamespace(rows=R, cols=C)
            if kind == "fwd":
                w = torch.randn(R, C, generator=gen, device="cuda") * 0.02
                w *= torch.exp(torch.randn(R, 1, generator=gen, device="cuda"))
                g = torch.rand(R, generator=gen, device="cuda") * 1.5 + 0.5
                out = torch.empty(R, C, dtype=torch.bfloat16, device="cuda")
                tab = (ds.ds_wseg * 1)(ds.WSeg(w=w, gain=g, w_eff=out).to_c())
                fns.append(lambda st, t=tab: lib.ds_wn_forward(t, 1, ds.DS_BF16, eps, st))
                self.keep += [w, g, out]
                self.bytes[name] = R * C * (4 + 2) + R * 4
                op = ds.DS_OP_WN_FORWARD
            else:
                x = torch.randn(R, C, generator=gen, device="cuda").to(torch.bfloat16)
                r = torch.randn(R, C, generator=gen, device="cuda").to(torch.bfloat16)
                al = torch.randn(C, generator=gen, device="cuda") * 0.05
                h = torch.empty_like(x)
                tab = (ds.ds_aseg * 1)(ds.ASeg(x=x, r=r, y=h, alpha=al).to_c())
                fns.append(lambda st, t=tab: lib.ds_slerp_rows(t, 1, eps, st))
                self.keep += [x, r, al, h]
                self.bytes[name] = call_bytes("slerp", act=act)
                op = ds.DS_OP_SLERP_ROWS
            self.rows[name] = R
            self.tables.append(tab)
            p, grp, cl = ds.ds_row_class(op, C)
            self.classes[name] = {ds.DS_PATH_CLUSTER: f"cluster of {cl} CTAs", ds.DS_PATH_TWO_PASS:
                                  f"two-pass stream, {cl} CTAs per row"}.get(p, f"staged ({grp} threads per row)")
        self.calls = [fns]
        self.inputs, self.outputs = [], []

    def run(self, stream_ptr: int, events=None, k: int = 0) -> None:
        Step.run(self, stream_ptr, events, k)


def time_calls(step, K: int, W: int, sp: int) -> dict[str, float]:
    """Mean CUDA-event time (ms) of each call of `step` over K timed steps
    after W warm-up steps (calls run in the step's order, so each call's
    inputs were pushed out of L2 by the calls between two uses)."""
    import torch

    for k in range(W):
        step.run(sp, None, k)
    torch.cuda.synchronize()
    n = len(step.names)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(K)]
    for k in range(K):
        step.run(sp, evs[k], k)
    torch.cuda.synchronize()
    return {name: statistics.fmean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(K))
            for i, name in enumerate(step.names)}


EXTRA_CONFIGS = ("wide", "long_rows", "optimizer", "act_backward", "dory", "gain", "mlp_pair")


def extra_calls(seed: int, K: int, sp: int, peak: float) -> dict:
    """Every other workload's calls, each call timed on its own (CUDA events,
    mean over K steps after 3 warm-up steps) and reported against the HBM
    peak; not part of the step's `value`.  The L2-resident MLP pair also
    reports its calls replayed from one CUDA graph."""
    import torch

    from l2_row_b200 import ds

    out = {}
    for label in EXTRA_CONFIGS:
        st = LongRows(seed) if label == "long_rows" else Step(seed=seed, config=label)
        ms = time_calls(st, K, 3, sp)
        if ds.ds_get_device_status(sp) != ds.DS_OK:
            raise RuntimeError(f"device error in the {label} calls")
        calls = {}
        for name in st.names:
            t_s = ms[name] * 1e-3
            gbs = st.bytes[name] / t_s / 1e9
            calls[name] = {"us": round(ms[name] * 1e3, 2), "bytes": st.bytes[name], "gb_s": round(gbs, 1),
                           "frac_of_peak": round(gbs / peak, 4), "rows_s": round(st.rows[name] / t_s, 1)}
            if isinstance(st, LongRows):
                calls[name]["class"] = st.classes[name]
        out[label] = {"workload": WORKLOADS[label], "steps": K, "calls": calls}
        if st.copies > 1:
            gms = graph_replay_ms(st)
            total = sum(st.bytes.values())
            out[label]["graph"] = {"ms_per_step": round(gms, 5), "gb_s": round(total / (gms * 1e-3) / 1e9, 1),
                                   "calls_per_replay": st.copies * len(st.names)}
        del st
        torch.cuda.empty_cache()
    return out


def graph_replay_ms(step: Step, reps: int = 20) -> float:
    """Per-step time of the calls replayed from one CUDA graph that holds one
    step on each buffer copy (launch-bound workloads)."""
    import torch

    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        for k in range(step.copies):
            step.run(side.cuda_stream, None, k)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * step.copies)
    del g
    return ms


def run_ours(args, rank: int, world: int, local_rank: int) -> None:
    import torch

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        dist = dist_mod

    from l2_row_b200 import ds

    step = LongRows(rank) if args.config == "long_rows" else Step(seed=rank, config=args.config)
    names = step.names
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    bytes_per, rows_per = step.bytes, step.rows
    step_total = sum(bytes_per.values())

    for k in range(max(3, args.warmup)):
        step.run(sp, None, k)
    torch.cuda.synchronize()
    if ds.ds_get_device_status(sp) != ds.DS_OK:
        raise RuntimeError("device error during warm-up")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    n0 = ds.ds_launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for k in range(K):
            step.run(sp, evs[k], k)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches = ds.ds_launch_count() - n0
    if ds.ds_get_device_status(sp) != ds.DS_OK:
        raise RuntimeError("device error in the timed region")

    total_ms = evs[0][0].elapsed_time(evs[-1][-1])
    per_call = {name: [evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(K)] for i, name in enumerate(names)}
    t = max_over_ranks(dist, [total_ms] + [statistics.fmean(per_call[n]) for n in names], "cuda")
    total_ms = t[0]
    call_ms = {name: t[i + 1] for i, name in enumerate(names)}

    ms_per_step = total_ms / K
    value = whole_job_gbs(world, step_total, ms_per_step)

    peak, peak_src = measured_peaks()
    kernels = {}
    for name in names:
        t_s = call_ms[name] * 1e-3
        gbs = bytes_per[name] / t_s / 1e9
        kernels[name] = {"us": round(call_ms[name] * 1e3, 2), "bytes": bytes_per[name], "gb_s": round(gbs, 1),
                         "frac_of_peak": round(gbs / peak, 4), "rows_s": round(rows_per[name] / t_s, 1)}
    fwd_bwd = None
    fw = [n for n, k, _ in step.plan if k == "fwd"]
    bw = [n for n, k, _ in step.plan if k == "bwd"]
    if fw and bw:
        fb_t = sum(call_ms[n] for n in fw + bw) * 1e-3
        fb_b = sum(bytes_per[n] for n in fw + bw)
        fwd_bwd = {"gb_s": round(fb_b / fb_t / 1e9, 1), "rows_s": round(sum(rows_per[n] for n in fw) / fb_t, 1),
                   "frac_of_peak": round(fb_b / fb_t / 1e9 / peak, 4)}
    dom = max(names, key=lambda n: call_ms[n])
    ach = bytes_per[dom] / (call_ms[dom] * 1e-3) / 1e9
    traffic = recorded_traffic(f"ds_{dom}") if args.config == "step" else None
    roofline = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                "frac": round(ach / peak, 4), "traffic": traffic, "kernel": f"ds_{dom}",
                "algorithmic_bytes": bytes_per[dom], "peak_source": peak_src}

    graph = None
    if step.copies > 1:
        gms = graph_replay_ms(step)
        graph = {"ms_per_step": round(gms, 5), "gb_s": round(step_total / (gms * 1e-3) / 1e9, 1),
                 "calls_per_replay": step.copies * len(names)}

    e2e = None
    if not args.no_e2e and step.inputs:
        e2e = measure_e2e(step, args.e2e_steps, step_total, sp, world, dist)

    extras = None
    if args.config == "step" and world == 1 and not args.no_extras:
        extras = extra_calls(rank, max(5, min(args.steps, 20)), sp, peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "step":
        cpu = cpu_baseline(step)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    l2_note = ("no flush: every call reads > 126 MB and consecutive calls touch disjoint buffers"
               if step.copies == 1 else
               f"no flush: each step uses the next of {step.copies} buffer copies "
               f"({step.copies * step_total / 1e6:.0f} MB > 126 MB L2)")
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded, host-generated)",
        "config": {"workload": WORKLOADS[args.config], "eps": EPS, "bytes_per_step": step_total, "l2": l2_note,
                   "parallelism": f"replicas x{world} (rows are independent; no collective)"},
        "kernels": kernels, "fwd_bwd": fwd_bwd, "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": launches, "clocks": clocks.summary(),
    }
    if graph:
        line["graph"] = graph
    if extras:
        line["extras"] = extras
    print(json.dumps(line), flush=True)


def measure_e2e(step: Step, steps: int, step_total: int, sp: int, world: int, dist) -> dict:
    """The same step through the C ABI starting from pinned host buffers:
    every step copies its inputs host -> device, runs the calls and copies
    every output back.  The copies run on two streams of their own, so that
    step k's outputs go back while step k + 1's inputs come in (PCIe is full
    duplex): the inputs wait for the previous step's calls, the calls wait
    for their inputs and for the previous step's outputs to be read."""
    import torch

    def pin(d, a):
        h = torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
        return h.view(torch.bfloat16) if d.dtype == torch.bfloat16 else h

    h_in = [(d, pin(d, a)) for d, a in step.inputs]
    outs = step.outputs
    h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(d.numel() * d.element_size() for d, _ in h_in)
    d2h = sum(o.numel() * o.element_size() for o in outs)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    done = torch.cuda.Event()      # the step's calls finished (inputs free, outputs ready)
    got_in = torch.cuda.Event()    # the step's inputs arrived
    sent_out = torch.cuda.Event()  # the step's outputs were read back (outputs free)
    done.record(comp)
    sent_out.record(comp)

    def one():
        s_in.wait_event(done)
        with torch.cuda.stream(s_in):
            for d, h in h_in:
                d.copy_(h, non_blocking=True)
        got_in.record(s_in)
        comp.wait_event(got_in)
        comp.wait_event(sent_out)
        step.run(sp)
        done.record(comp)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            for o, h in zip(outs, h_out):
                h.copy_(o, non_blocking=True)
        sent_out.record(s_out)

    one()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for _ in range(steps):
        one()
    comp.wait_event(sent_out)
    b.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, [a.elapsed_time(b) / steps], "cuda")[0]
    return {"value": round(whole_job_gbs(world, step_total, ms), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "overlap": "inputs of step k + 1 in while outputs of step k go out (two copy streams)"}


# ------------------------------------------------------- the CPU oracle ----

def oracle_sample(model_weights, act, frac: float):
    """A bounded slice of the step: the first `frac` of every weight
    segment's rows and of the activation rows."""
    from l2_row_b200 import workloads as wl

    segs = []
    for s in model_weights:
        n = max(1, int(round(s.rows * frac)))
        segs.append(wl.WeightSeg(s.name, s.w[:n], s.g[:n], s.gy[:n]))
    n = max(1, int(round(act.rows * frac)))
    a = wl.ActRows(act.name, act.x[:n], act.r[:n], act.alpha)
    return segs, a


def time_oracle_step(segs, a, nthreads: int) -> tuple[float, int]:
    """Run the six operations of a step on the oracle; (seconds, bytes)."""
    import oracle

    t0 = time.perf_counter()
    for s in segs:
        oracle.wn_forward(s.w, s.g, eps=EPS, nthreads=nthreads)
    oracle.l2_rows(a.x, None, eps=EPS, nthreads=nthreads)
    for s in segs:
        oracle.wn_backward(s.w, s.gy, s.g, eps=EPS, nthreads=nthreads)
    oracle.l2_rows(a.x, a.r, eps=EPS, nthreads=nthreads)
    for s in segs:
        oracle.row_renorm(s.w, eps=EPS, nthreads=nthreads)
    oracle.slerp_rows(a.x, a.r, a.alpha, eps=EPS, nthreads=nthreads)
    dt = time.perf_counter() - t0
    b = step_bytes(segs, a.rows, a.cols)
    return dt, sum(b.values())


def cpu_baseline(step: Step, min_seconds: float = 10.0, max_reps: int = 20) -> dict:
    """The oracle on the host cores over the whole step's inputs, repeated
    until at least `min_seconds` of work (bounded by `max_reps`)."""
    import oracle

    cores = oracle.default_threads()
    segs, a = oracle_sample(step.wg["model"], step.ag["x"], 1.0)
    total, nbytes, reps = 0.0, 0, 0
    while reps < max_reps and (reps == 0 or total < min_seconds):
        dt, b = time_oracle_step(segs, a, cores)
        total += dt
        nbytes += b
        reps += 1
    # the same oracle on one thread, over the first 1/16 of every segment's
    # and of the activation rows (about a second)
    s1, a1 = oracle_sample(step.wg["model"], step.ag["x"], 1.0 / 16)
    dt1, b1 = time_oracle_step(s1, a1, 1)
    return {"value": round(nbytes / total / 1e9, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"the whole step (all six calls on every weight segment and all activation rows, "
                      f"{nbytes / reps / 1e6:.0f} MB algorithmic) x {reps}, {total:.1f} s wall",
            "single_thread": {"value": round(b1 / dt1 / 1e9, 3), "unit": "GB/s", "cores": 1,
                              "sample": f"the first 1/16 of every segment's rows and of the activation rows "
                                        f"({b1 / 1e6:.0f} MB algorithmic) x 1, {dt1:.1f} s wall"}}


def run_reference(args, rank: int, world: int) -> None:
    """The reference arm: the float64 oracle as it stands, on the host cores,
    same metric and workload; each step runs the six calls over the whole
    step's inputs (every weight segment, every activation row), as the
    cpu_baseline leg does."""
    if rank != 0:
        return
    import oracle
    from l2_row_b200 import workloads as wl

    model = wl.whole_model(0)
    act = wl.activations(0, ACT_ROWS, ACT_COLS).acts[0]
    cores = oracle.default_threads()
    segs, a = oracle_sample(model.weights, act, 1.0)
    for _ in range(max(1, args.warmup)):
        time_oracle_step(segs, a, cores)
    total, nbytes = 0.0, 0
    for _ in range(args.steps):
        dt, b = time_oracle_step(segs, a, cores)
        total += dt
        nbytes += b
    value = nbytes / total / 1e9
    sample = (f"the whole step per timed step (all six calls on every weight segment and all activation rows, "
              f"{nbytes / args.steps / 1e6:.0f} MB algorithmic) x {args.steps}, {total:.1f} s wall")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, host-generated)",
        "config": {"workload": WORKLOAD, "eps": EPS, "sample": sample},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
