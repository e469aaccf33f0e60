"""Plain fp64 CPU oracle of the HARD-KV decode step (test infrastructure only)."""
