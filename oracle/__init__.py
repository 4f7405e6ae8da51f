"""CPU oracle (test infrastructure only; see uw_oracle)."""
