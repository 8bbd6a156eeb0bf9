"""FlashCart-style irreducible-Cartesian tensor products on NVIDIA B200.

The compute lives in the CUDA library ``libflashcart.so`` (C ABI, declared in
``include/flashcart.h``); ``cartesian_tensor_products_b200.flashcart`` is the
thin ctypes binding over it.  ``workloads`` draws the seeded inputs.
Nothing is imported eagerly so that the input generators can be used on a
machine without the built library.
"""
__all__ = ["flashcart", "workloads"]
