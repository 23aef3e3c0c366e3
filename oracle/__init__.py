"""CPU oracle (test infrastructure only; see twell_oracle.py)."""
