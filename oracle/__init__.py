"""fp64 CPU oracle for the ECASQ solver. Test infrastructure only (see oracle.py)."""
