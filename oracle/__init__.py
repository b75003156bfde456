"""fp64 CPU oracle (test infrastructure only; see tq_oracle.py)."""
from .tq_oracle import *  # noqa: F401,F403
from . import tq_oracle  # noqa: F401
