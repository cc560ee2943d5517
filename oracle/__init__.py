"""CPU oracle (test infrastructure only; see nvium_oracle's header)."""
from .nvium_oracle import *  # noqa: F401,F403
