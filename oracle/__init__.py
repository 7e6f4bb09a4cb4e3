"""CPU oracle for the RotateAttention INT4 attention forward (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg use this
package.  It is independent of the CUDA library: it does not import it and
shares no code with it.
"""
from .oracle import *  # noqa: F401,F403
