"""CPU oracle for the AWQ scale search: test infrastructure only (see awq_oracle.py)."""
from . import awq_oracle  # noqa: F401
