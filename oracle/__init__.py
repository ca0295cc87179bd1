"""CPU oracle for block-sparse video attention -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library and never
imports it.
"""
