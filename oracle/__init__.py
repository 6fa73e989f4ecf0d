"""Float64 CPU oracle of the TurboQuant hot path (test infrastructure only)."""
