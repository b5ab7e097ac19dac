"""Float64 CPU oracle for the selective state update (test infrastructure only)."""
