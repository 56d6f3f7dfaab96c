"""fp64 CPU oracle of tree-indexed sparse attention (test infrastructure only)."""
