"""CPU oracle for the 8-bit quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg (and its reference arm) may import this package.  The
product path (the CUDA library and its Python binding) never imports, links or runs
anything here, and this package imports nothing from the product.
"""
from .oracle import *  # noqa: F401,F403
