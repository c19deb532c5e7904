"""fp64 CPU oracle for the CRISP sparse-prefill path (test infrastructure only)."""
from . import crisp_oracle  # noqa: F401
