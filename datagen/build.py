"""Compile the GPU side of the seeded input generator into datagen/libdatagen.so."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "fill.cu")
LIB = os.path.join(HERE, "libdatagen.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # one temporary per process: ranks that build at the same time do not share a file
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = [os.environ.get("NVCC", "nvcc"), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           SRC, "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)  # atomic: a loader never sees a partial file
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
