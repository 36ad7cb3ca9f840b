"""CPU oracle (test infrastructure only): plain float64 statement of the method.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use it.
"""
from .tq_oracle import *  # noqa: F401,F403
from .tq_oracle import __all__  # noqa: F401
