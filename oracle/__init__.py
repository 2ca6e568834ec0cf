"""CPU oracle for AQUA (test infrastructure only; see aqua_oracle's header)."""
from .aqua_oracle import *  # noqa: F401,F403
from . import aqua_oracle  # noqa: F401
