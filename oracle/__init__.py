"""fp64 CPU oracle of the GQE forward pass (test infrastructure only)."""
