"""CPU oracle (test infrastructure only): see bsa_oracle."""
from . import bsa_oracle  # noqa: F401
