"""Float64 CPU oracle (test infrastructure only; see encoder_oracle.py)."""
