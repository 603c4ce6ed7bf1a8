"""Float64 CPU oracle of the TTT layer (test infrastructure; see ttt_oracle.py)."""
from .ttt_oracle import *  # noqa: F401,F403
from .ttt_oracle import __all__  # noqa: F401
