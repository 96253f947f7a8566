"""CPU float64 oracle (test infrastructure only; see rbs_oracle's header)."""

from . import rbs_oracle  # noqa: F401
