"""fp64 CPU oracle of the DM0 merged-attention hot path (test infrastructure only)."""
