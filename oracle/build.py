"""Compile the plain-C oracle into ``oracle/_build/liboracle.so``.

Test infrastructure: the oracle is built so that the tests, the smoke check
and the benchmark's CPU-baseline leg can call it.  Building it is not using it;
the CUDA library never links or loads it.

Flags: -O2, no fast-math (IEEE semantics, so fp64 results are reproducible),
OpenMP over independent query rows.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "paged_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "liboracle.so")

CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile ``src`` to the shared object ``out`` (skipped when up to date)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
