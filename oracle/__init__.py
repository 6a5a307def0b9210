"""CPU oracle for the Gated DSA layer (test infrastructure only; see oracle.py)."""
