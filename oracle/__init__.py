"""fp64 CPU oracle of the Dual-QK decode path (test infrastructure only)."""
