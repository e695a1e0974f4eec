"""CPU fp64 oracle (test infrastructure; see tq_oracle.py for what may import it)."""
from .tq_oracle import *  # noqa: F401,F403
from .tq_oracle import GROUP  # noqa: F401
