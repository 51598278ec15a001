"""fp64 CPU oracle (test infrastructure only; see kvc_oracle.py)."""
from . import kvc_oracle  # noqa: F401
