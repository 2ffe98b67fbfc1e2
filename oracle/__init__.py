"""CPU oracle of the OmniQuant fake-quantized linear calibration step (test infrastructure)."""
