"""CPU oracle (test infrastructure only; see kivi_oracle's module docstring)."""
