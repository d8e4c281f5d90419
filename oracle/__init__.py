"""fp64 CPU oracle (test infrastructure only; see gptq_oracle.py)."""
