"""CPU oracle of the wave-round hot path (test infrastructure only)."""
