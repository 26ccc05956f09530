"""Compile the float64 CPU oracle (test infrastructure) into oracle/liblsa_oracle.so."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lsa_oracle.c")
LIB = os.path.join(HERE, "liblsa_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # one temporary per process: ranks that build at the same time do not share a file
    tmp = f"{LIB}.{os.getpid()}.tmp"
    # -ffp-contract=off: every multiply and add rounds on its own, as written.
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           SRC, "-o", tmp, "-lm"]
    try:
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)  # atomic: a loader never sees a partial file
    finally:
        if os.path.exists(tmp):  # a failed compile leaves no temporary behind
            os.remove(tmp)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
