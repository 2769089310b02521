"""fp64 CPU oracle of the BasisKV decode step (test infrastructure only)."""
from . import basiskv_oracle  # noqa: F401
