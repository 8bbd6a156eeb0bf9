"""FP64 CPU reference ("oracle") for the FlashCart tensor-product hot path.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
CPU-baseline leg of the benchmark, never by the product library.
"""
