"""CPU oracle of the Hymba hybrid-head mixer (test infrastructure only; see hymba_oracle)."""
from .hymba_oracle import *  # noqa: F401,F403
from . import hymba_oracle  # noqa: F401
