"""Build the sm_100a CUDA library liblsa_b200.so in-tree (nvcc, no GPU needed)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liblsa_b200.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(p) for p in _deps() + [__file__])
        if os.path.getmtime(LIB) >= newest:
            return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    # one temporary per process: ranks that build at the same time do not share a file
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = [nvcc, "-shared", *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, *_sources(),
           "-o", tmp]
    if verbose:
        print(" ".join(cmd))
    try:
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)  # atomic: a loader never sees a partial file
    finally:
        if os.path.exists(tmp):  # a failed compile leaves no temporary behind
            os.remove(tmp)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None))
