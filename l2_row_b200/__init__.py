"""l2_row_b200 -- per-row L2 normalisation of weight and activation rows on B200.

The compute path is the C-ABI library ``libds.so`` (hand-written CUDA for
sm_100a, built from ``csrc/``); ``l2_row_b200.ds`` is its thin ctypes binding
with the same call names.  Importing the binding raises if the library was not
built: there is no CPU fallback.
"""
from __future__ import annotations

__all__ = ["ds", "workloads"]


def __getattr__(name):
    import importlib

    if name in ("ds", "workloads"):
        return importlib.import_module(f"{__name__}.{name}")
    if name.startswith("ds_") or name in ("WSeg", "ASeg", "DSError"):
        return getattr(importlib.import_module(f"{__name__}.ds"), name)
    raise AttributeError(name)
