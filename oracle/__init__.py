"""CPU oracle of HSTU pointwise attention (float64).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library.
"""
