"""CPU oracle for the DSA hot path (test infrastructure only; see oracle.py)."""
