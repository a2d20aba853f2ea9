"""Float64 CPU oracle (test infrastructure only; see fldce_oracle.py)."""
from .fldce_oracle import *  # noqa: F401,F403
