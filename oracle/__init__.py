"""CPU oracle (test infrastructure only; see awq_oracle.py's header)."""
