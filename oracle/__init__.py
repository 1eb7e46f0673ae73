"""CPU oracle (test infrastructure only; see lsa_oracle)."""
from .lsa_oracle import *  # noqa: F401,F403
from . import lsa_oracle  # noqa: F401
