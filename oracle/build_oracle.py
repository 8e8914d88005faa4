"""Compile the C host oracle (oracle/c/) into oracle/c/libbitssm_oracle.so.

Test infrastructure: called by tests/ (through oracle.c_oracle) and by
__graft_entry__.build().  gcc, -O2, -ffp-contract=off (every a * b + c of the
source stays two rounded operations), OpenMP over independent rows."""

from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "c", "bitssm_oracle.c")
HDR = os.path.join(HERE, "c", "bitssm_oracle.h")
LIB = os.path.join(HERE, "c", "libbitssm_oracle.so")


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR), os.path.getmtime(__file__))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
