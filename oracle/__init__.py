"""Float64 CPU oracle for the p4 EQ-Linear layer (test infrastructure only)."""
