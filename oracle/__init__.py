"""CPU oracle for the Twilight decode path (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
arm import this package.  The CUDA library never calls it and shares no code
with it.
"""
from .twilight_oracle import *  # noqa: F401,F403
