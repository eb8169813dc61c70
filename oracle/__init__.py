"""fp64 CPU oracle for causal linear attention -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
