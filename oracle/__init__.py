"""Float64 CPU oracle for the DSA step: test infrastructure only (see dsa_oracle)."""
from .dsa_oracle import *  # noqa: F401,F403
