"""CPU oracle (test infrastructure only; see ptl_oracle)."""
