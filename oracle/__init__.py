"""fp64 CPU oracle of the MC-Sparse hot path (test infrastructure only)."""
