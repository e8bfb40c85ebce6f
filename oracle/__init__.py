"""CPU oracle (test infrastructure only; see sla_oracle.py)."""
