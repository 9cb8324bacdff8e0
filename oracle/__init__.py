"""CPU oracle of the compressed-KV decode step.  Test infrastructure only."""
