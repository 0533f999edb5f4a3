"""fp64 CPU oracle of the sparse-attention hot path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package.  It shares no code with the CUDA library.
"""
from .lsa_oracle import *  # noqa: F401,F403
