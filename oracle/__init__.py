"""fp64 CPU oracle of the HySparse2 hybrid sparse attention step (test infrastructure only)."""
from .hs2_oracle import *  # noqa: F401,F403
