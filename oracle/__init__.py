"""fp64 CPU oracle for MLA decode -- test infrastructure only.

Only the tests, the package entry's smoke check and the benchmark's CPU
baseline leg may import this package; the product path never does.
"""
