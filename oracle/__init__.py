"""fp64 CPU oracle of the DeepSeekMoE layer forward pass (test infrastructure only)."""
