"""Float64 CPU oracle (test infrastructure; see vdn_oracle.py's header)."""
from .vdn_oracle import *  # noqa: F401,F403
