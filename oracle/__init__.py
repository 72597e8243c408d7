"""Plain CPU oracle for the codebook-VQ linear layer (test infrastructure only)."""
