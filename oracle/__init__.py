"""fp64 CPU oracle (test infrastructure; see ds4a_oracle)."""
