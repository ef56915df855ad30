"""fp64 CPU oracle for the chunked TTT-layer forward pass (test infrastructure only)."""
