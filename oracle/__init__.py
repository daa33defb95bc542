"""CPU oracle (test infrastructure; see msa_oracle's header for who may import it)."""
from . import msa_oracle  # noqa: F401
