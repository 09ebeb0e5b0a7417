"""Compile the fp64 CPU oracle (oracle.c) into a shared library with gcc.

Test infrastructure only.  Flags keep IEEE fp64 semantics: no fast-math and no FMA
contraction, so every sum is the sequential sum the source writes.

Two builds of the same source: liboracle.so (one thread; what the tests use) and
liboracle_omp.so (-fopenmp: the independent row and element loops split over the host's
cores, dot products still sequential, so its results are bit-identical), which only the
benchmark's CPU baseline times.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
LIB_OMP = os.path.join(HERE, "liboracle_omp.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
          "-Wall", "-Wextra", "-Wno-unused-parameter", "-Wno-unknown-pragmas"]


def build(src: str = SRC, out: str = LIB, extra: tuple[str, ...] = (), force: bool = False) -> str:
    """Build ``src`` into ``out`` unless ``out`` is newer than ``src``; return ``out``."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)
            and os.path.getmtime(out) >= os.path.getmtime(__file__)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_omp(force: bool = False) -> str:
    """The OpenMP build of the same source (all host cores; bit-identical results)."""
    return build(out=LIB_OMP, extra=("-fopenmp",), force=force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    print(build_omp(force="--force" in sys.argv))
