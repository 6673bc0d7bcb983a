"""fp64 CPU oracle (test infrastructure only; see opr_oracle's header)."""

from .opr_oracle import *  # noqa: F401,F403
