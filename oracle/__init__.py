"""fp64 CPU oracle (test infrastructure only; see hyb_oracle.py)."""
from .hyb_oracle import *  # noqa: F401,F403
