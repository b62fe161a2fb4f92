"""CPU fp64 oracle (test infrastructure only; see qmoe_oracle.py)."""
from .qmoe_oracle import *  # noqa: F401,F403
