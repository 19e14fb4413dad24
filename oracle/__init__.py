"""NVFP4 CPU oracle -- test infrastructure.

Only the tests, the package smoke check and the benchmark's CPU-baseline and
reference legs may import this package.  The product path (the CUDA library
and its Python binding) never imports it and has no CPU fallback.
"""
from .oracle import *  # noqa: F401,F403
