"""CPU oracle of the GKDT detection head (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. The product path (the CUDA library and its binding)
never imports it, and it imports nothing from the product package.
"""
