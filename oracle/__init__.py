"""CPU oracle for the HHR decode-time retrieval path (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the benchmark's CPU-baseline / reference
arm may import this package.  It shares no code with the CUDA library.
"""
