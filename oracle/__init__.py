"""CPU oracle of the GSA layer (test infrastructure only; see gsa_oracle.py)."""
from .gsa_oracle import *  # noqa: F401,F403
