"""CPU oracle (fp64) of the decode-time coarse-to-fine retrieval path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path. It shares no code
with the CUDA implementation. Every function cites the page passage it follows.
"""
from .hhr_oracle import *  # noqa: F401,F403
from . import hhr_oracle  # noqa: F401
