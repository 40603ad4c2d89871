"""CPU oracle of the product-key memory layer (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library shares no code with it.
"""
