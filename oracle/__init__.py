"""CPU oracle of the DFlash draft step (test infrastructure only)."""
