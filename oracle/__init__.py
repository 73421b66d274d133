"""CPU oracle of the IndexMem hot path (test infrastructure; never on the product path)."""
from .indexmem_oracle import *  # noqa: F401,F403
