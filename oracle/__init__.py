"""fp64 CPU oracle of the CSA forward path (test infrastructure, see csa_oracle.py)."""
from .csa_oracle import *  # noqa: F401,F403
