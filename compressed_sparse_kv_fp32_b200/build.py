"""Build step of the CUDA library: nvcc for sm_100a, in-tree, no JIT cache.

    python -m compressed_sparse_kv_fp32_b200.build
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIBRARY = os.path.join(HERE, "libadamas.so")
MAIN_SOURCE = os.path.join(HERE, "csrc", "adamas.cu")
HEADER = os.path.join(ROOT, "include", "adamas.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) +
                  glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [HEADER])


def stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/adamas.cu into libadamas.so next to this file."""
    if not force and not stale():
        return LIBRARY
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, MAIN_SOURCE]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
