"""CPU oracle for the nanochat forward pass (test infrastructure only)."""
