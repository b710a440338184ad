"""fp64 CPU oracle for the NSA forward pass -- test infrastructure only (see oracle.py)."""
