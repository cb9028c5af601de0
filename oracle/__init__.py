"""fp64 CPU oracle (test infrastructure only; see svdq_oracle's module docstring)."""
