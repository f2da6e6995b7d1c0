"""fp64 CPU oracle for the NVFP4 W4A16 MoE FFN layer (test infrastructure only)."""
