"""CPU oracle for the Wan 2.1 DiT hot path (test infrastructure only; see wan_oracle)."""
from .wan_oracle import *  # noqa: F401,F403
from . import wan_oracle  # noqa: F401
