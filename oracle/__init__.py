"""CPU oracle for the rotated W4A4 linear layer (test infrastructure only).

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg import this package; the CUDA library never does."""
