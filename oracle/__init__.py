"""CPU float64 oracle (test infrastructure; never on the product path)."""
from .tpla_oracle import *  # noqa: F401,F403
