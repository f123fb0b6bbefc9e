"""fp64 CPU oracle (test infrastructure only; see mla_oracle's module docstring)."""
from .mla_oracle import *  # noqa: F401,F403
from .mla_oracle import Dims, Weights  # noqa: F401
