"""CPU oracle (test infrastructure only; see rdt_oracle's header)."""
from . import rdt_oracle  # noqa: F401
