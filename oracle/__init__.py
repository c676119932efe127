"""CPU oracle (test infrastructure only; see dg_oracle's header for who may use it)."""
from .dg_oracle import *  # noqa: F401,F403
from . import dg_oracle  # noqa: F401
