"""CPU float64 oracle for AM-OMP KV compaction — test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py (cpu_baseline and the
reference arm) may import this package; the CUDA library never does.
"""
from .am_oracle import *  # noqa: F401,F403
