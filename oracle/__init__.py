"""CPU oracle (test infrastructure only; see whale_oracle.py)."""
