"""fp64 CPU oracle for STAR-KV-style low-rank, quantised KV-cache decode.

TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python binding)
never imports, calls or links anything here.
"""
from .starkv_oracle import *  # noqa: F401,F403
