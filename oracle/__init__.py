"""CPU float64 oracle (test infrastructure only; see sparvar_oracle.py)."""
from . import sparvar_oracle  # noqa: F401
