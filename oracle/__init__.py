"""Float64 CPU oracle for the ROCS forward (test infrastructure only; see rocs_oracle)."""
