"""Compile the fp64 CPU oracle (oracle.c) into a shared library with gcc.

Test infrastructure only.  Flags keep IEEE fp64 semantics: no fast-math and no FMA
contraction, so every sum is the sequential sum the source writes.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]


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


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
