"""CPU oracle for the MoE layer hot path (test infrastructure; never on the product path)."""
