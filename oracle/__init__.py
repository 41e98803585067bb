"""fp64 CPU oracle for the LittleBit layer (test infrastructure only)."""
