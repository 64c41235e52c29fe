"""CPU oracle package (test infrastructure only; see bitlinear_oracle.py)."""
