"""fp64 CPU oracle for the DSA hot path (test infrastructure only)."""
