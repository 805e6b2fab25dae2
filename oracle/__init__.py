"""CPU oracle package (test infrastructure only; see absp_oracle)."""
