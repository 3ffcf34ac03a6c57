"""Build step of the CUDA library: nvcc for sm_100a, in-tree, no JIT cache.

    python -m compressed_sparse_kv_fp32_b200.build [--force] [-v]

The library is csrc/adamas.cu (the C ABI, the key encoder, the distance dump)
plus csrc/decode_inst.cu compiled once per query-head group size (1..8) so that
the decode kernel's instances compile in parallel; the objects are linked into
libadamas.so next to this file.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIBRARY = os.path.join(HERE, "libadamas.so")
MAIN_SOURCE = os.path.join(HERE, "csrc", "adamas.cu")
DECODE_SOURCE = os.path.join(HERE, "csrc", "decode_inst.cu")
HEADER = os.path.join(ROOT, "include", "adamas.h")
GROUP_SIZES = range(1, 9)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC"]
NVCC_FLAGS = [*COMPILE_FLAGS, "-shared"]  # single-step build flags (kept for reference by tools)


def _sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) +
                  glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [HEADER])


def stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(s) > t for s in _sources())


def _run(cmd, verbose):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise subprocess.CalledProcessError(r.returncode, cmd)
    if verbose:
        sys.stderr.write(r.stderr)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the sources into libadamas.so next to this file (parallel nvcc per object)."""
    if not force and not stale():
        return LIBRARY
    nvcc = os.environ.get("NVCC", "nvcc")
    tag = f".tmp{os.getpid()}"
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose else []
    jobs = [[nvcc, *COMPILE_FLAGS, *extra, "-c", "-o", os.path.join(objdir, f"adamas{tag}.o"), MAIN_SOURCE]]
    for g in GROUP_SIZES:
        jobs.append([nvcc, *COMPILE_FLAGS, *extra, f"-DADAMAS_DECODE_G={g}", "-c",
                     "-o", os.path.join(objdir, f"decode_g{g}{tag}.o"), DECODE_SOURCE])
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        list(ex.map(lambda c: _run(c, verbose), jobs))
    objs = [j[j.index("-o") + 1] for j in jobs]
    tmp = os.path.join(HERE, f"libadamas{tag}.so")
    _run([nvcc, *ARCH, "-shared", "-o", tmp, *objs], verbose)
    os.replace(tmp, LIBRARY)
    for o in objs:
        os.remove(o)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
