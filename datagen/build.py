"""Compile the seeded input generator's native sides: the GPU fill (datagen/libdatagen.so,
nvcc, sm_100a) and the host slice regenerator (datagen/libdatagen_host.so, gcc + OpenMP)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "fill.cu")
LIB = os.path.join(HERE, "libdatagen.so")
HOST_SRC = os.path.join(HERE, "csrc", "normal_host.c")
HOST_LIB = os.path.join(HERE, "libdatagen_host.so")


def _compile(cmd_head: list, src: str, lib: str) -> str:
    # one temporary per process: ranks that build at the same time do not share a file
    tmp = f"{lib}.{os.getpid()}.tmp"
    try:
        subprocess.check_call(cmd_head + [src, "-o", tmp])
        os.replace(tmp, lib)  # atomic: a loader never sees a partial file
    finally:
        if os.path.exists(tmp):  # a failed compile leaves no temporary behind
            os.remove(tmp)
    return lib


def _fresh(src: str, lib: str) -> bool:
    return os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(src)


def build(force: bool = False) -> str:
    if not force and _fresh(SRC, LIB):
        return LIB
    cmd = [os.environ.get("NVCC", "nvcc"), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]
    return _compile(cmd, SRC, LIB)


def build_host(force: bool = False) -> str:
    if not force and _fresh(HOST_SRC, HOST_LIB):
        return HOST_LIB
    cmd = [os.environ.get("CC", "gcc"), "-shared", "-fPIC", "-O2", "-fvisibility=hidden",
           "-std=c11"]
    return _compile(cmd, HOST_SRC, HOST_LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_host(force="--force" in sys.argv))
