"""CPU oracle for the CLSA path (test infrastructure; see clsa_oracle.py)."""
