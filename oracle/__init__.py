"""fp64 CPU oracle (test infrastructure only; see bsa_oracle's header)."""
from . import bsa_oracle  # noqa: F401
