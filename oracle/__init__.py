"""fp64 CPU oracle of the Stem prefill hot path (test infrastructure only:
tests, the smoke check and the bench's CPU-baseline leg use it; the product
path never does)."""
