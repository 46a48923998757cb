"""CPU oracle for one MoE layer forward: test infrastructure only (see moe_oracle.py)."""
