"""fp64 CPU oracle of the DiT-MoE sparse expert layer (test infrastructure only)."""
