"""Build the retrieval library in-tree: nvcc -> hash_hierarchical_top_b200/libhhr.so (sm_100a).

Run ``python -m hash_hierarchical_top_b200.build`` (or call ``build()``). The
library is a single CUDA translation unit; nvcc cross-compiles it without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libhhr.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(ROOT, "include", "hhr.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libhhr.so if it is missing or older than any source; return its path."""
    if not force and os.path.exists(LIB):
        t_lib = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t_lib for s in sources()):
            return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    if os.path.exists("/usr/local/cuda/bin/nvcc") and nvcc == "nvcc":
        nvcc = "/usr/local/cuda/bin/nvcc"
    tmp = LIB + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, os.path.join(CSRC, "hhr_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
