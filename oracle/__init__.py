"""fp64 CPU oracle for block sparse attention (test infrastructure only; see bsa_oracle)."""
from .bsa_oracle import *  # noqa: F401,F403
from .bsa_oracle import Grid, NEG_INF  # noqa: F401
