"""fp64 CPU oracle for the GLQ compressed-weight linear layer.

TEST INFRASTRUCTURE ONLY: imported by the test-suite, the package entry
point's smoke check and the benchmark's CPU-baseline leg, never by the CUDA
library.
"""
