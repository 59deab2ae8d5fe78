"""Builds ``liboracle.so`` from ``vca_oracle.c`` with gcc (test infrastructure).

``python -m oracle.build`` compiles it; importing ``oracle`` builds on first use
when the library is missing or older than its source.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "vca_oracle.c")
HDR = os.path.join(HERE, "vca_oracle.h")
OUT = os.path.join(HERE, "liboracle.so")

# No fast-math, no FMA contraction: every fused multiply-add is an explicit fmaf.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    stale = (not os.path.exists(OUT) or
             os.path.getmtime(OUT) < max(os.path.getmtime(SRC), os.path.getmtime(HDR)))
    if force or stale:
        tmp = OUT + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
