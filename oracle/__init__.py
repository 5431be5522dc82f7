"""CPU oracle of the W4A4 linear layer (test infrastructure; see fq_oracle)."""
from . import fq_oracle  # noqa: F401
