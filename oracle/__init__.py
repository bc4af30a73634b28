"""fp64 CPU oracle for the KronQ layer path (test infrastructure only)."""
