"""CPU oracle for the MoE path: test infrastructure only (see oracle.py)."""
