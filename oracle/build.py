"""Compile the plain-C oracle (test infrastructure) into oracle/_build/liboracle.so.

Run as ``python oracle/build.py``; ``oracle.load()`` also calls :func:`build` when the
library is missing or older than its source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "aqnf4_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle.so")

# Plain IEEE arithmetic: no contraction into FMA, no fast-math, default rounding.
CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    """Compile the oracle if needed and return the path of the shared library."""
    stale = force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC)
    if stale:
        os.makedirs(OUT_DIR, exist_ok=True)
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
