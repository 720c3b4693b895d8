"""Build the CPU oracle (plain C, fp64) into oracle/liboracle.so with gcc.

Test infrastructure only: tests/, __graft_entry__ and bench.py's CPU-baseline
leg load it. No fast-math and no floating-point contraction, so every
operation rounds as written in the source.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "q4g_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False, verbose: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "q4g_oracle.h"),
            os.path.join(HERE, "..", "datagen", "q4g_datagen.h")]
    if not force and os.path.exists(OUT) and all(
            os.path.getmtime(OUT) >= os.path.getmtime(d) for d in deps):
        return OUT
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-o", OUT + ".tmp", SRC, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
