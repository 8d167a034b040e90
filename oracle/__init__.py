"""CPU float64 oracle for the DPO head path (test infrastructure only; see dpo_oracle)."""
