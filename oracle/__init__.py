"""CPU oracle for the NVFP4 linear layer (test infrastructure; see nvfp4_oracle)."""
