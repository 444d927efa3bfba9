"""fp64 CPU oracle for the ConvKV Memory attention step (test infrastructure only)."""
