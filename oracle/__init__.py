"""fp64 CPU oracle for the Velox routed-attention path (test infrastructure only)."""
