"""fp64 CPU oracle of the HSTU jagged layer (test infrastructure; never used by the library)."""
from .hstu_oracle import *  # noqa: F401,F403
