"""fp64 CPU oracle of the HiLS attention forward pass (test infrastructure only)."""
