"""B200-native coarse-to-fine key retrieval for top-k sparse attention at decode time.

HHR (Geometry-Aware Key Routing page bounds + Learned Hash Projection Hamming
ranking) and the HISA indexer variant (block filter + token refinement), as
hand-written sm_100a CUDA kernels behind the C ABI in include/hhr.h.
"""
from . import hhr  # noqa: F401
from .hhr import HHRError, make_dims  # noqa: F401
from .step import DecodeStep, LayerCache  # noqa: F401
