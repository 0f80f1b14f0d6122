"""float64 CPU oracle for per-row L2 normalisation -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__ and the benchmark's
CPU-baseline leg (and its reference arm) may import this package.  The product
path (l2_row_b200) never does.  See oracle.h for the definitions and sources.
"""
from .oracle import *  # noqa: F401,F403
