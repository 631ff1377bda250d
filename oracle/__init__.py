"""fp64 CPU oracle for DCA (test infrastructure only; see dca_oracle)."""
from . import dca_oracle  # noqa: F401
