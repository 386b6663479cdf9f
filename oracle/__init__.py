"""fp64 CPU oracle of the GPTQ layer solver (test infrastructure only)."""
