"""CPU fp64 oracle for Sol-Attn (test infrastructure only; see sol_attn_oracle)."""
