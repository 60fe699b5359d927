"""fp64 CPU oracle (test infrastructure only; see mla_oracle.py)."""
