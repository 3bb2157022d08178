"""CPU oracle for the quantized linear layer (test infrastructure only)."""
