"""fp64 CPU oracle for the mixer hot path. TEST INFRASTRUCTURE ONLY (see oracle.py)."""
