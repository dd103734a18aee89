"""fp64 CPU oracle for the Sol-Attn forward — test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and reference
legs may import this package.  The product path never does.
"""
from .sol_attn_oracle import *  # noqa: F401,F403
