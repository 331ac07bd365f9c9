"""Token-level sparse attention with PDDP query grouping (MC-Sparse) on B200."""
