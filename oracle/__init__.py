"""CPU oracle of the sparse MoE layer forward pass (test infrastructure only;
never imported by the product path)."""
