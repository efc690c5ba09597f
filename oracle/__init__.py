"""CPU oracle package (test infrastructure only; see tri_oracle)."""
