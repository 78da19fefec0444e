"""Float64 CPU oracle for SAS gated block-sparse attention (test infrastructure only)."""
from . import sas_oracle  # noqa: F401
