"""fp64 CPU oracle of the MoE layer. Test infrastructure only (see moe_oracle)."""
