"""CPU oracle for the RotateAttention INT4 attention forward.

Test infrastructure only: the test suite, the package smoke check and the
benchmark's CPU-baseline leg may use it; the product path never does.
"""
