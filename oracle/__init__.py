"""fp64 CPU oracle (test infrastructure only; see mcs_oracle's header)."""
from .mcs_oracle import *  # noqa: F401,F403
from .mcs_oracle import POWER_ITERS, default_scale  # noqa: F401
