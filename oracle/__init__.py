"""CPU oracle (test infrastructure only; never imported by the library)."""
from .bsa_oracle import *  # noqa: F401,F403
from .bsa_oracle import Grid  # noqa: F401
