"""fp64 CPU oracle (test infrastructure only; see sda_oracle)."""
