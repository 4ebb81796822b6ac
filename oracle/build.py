"""Compile the plain-C oracle into ``oracle/libh3oracle.so`` with gcc.

Test infrastructure only (see ``oracle/__init__.py``).  The flags keep the
binary32 arithmetic plain IEEE: no fast-math, no contraction into FMA.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "h3_oracle.c")
LIB = os.path.join(HERE, "libh3oracle.so")

CFLAGS = ["-std=c99", "-O1", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra", "-Werror"]


def build(src: str = SRC, out: str = LIB, extra: list[str] | None = None) -> str:
    """Compile ``src`` into the shared library ``out`` and return its path."""
    cmd = ["gcc", *CFLAGS, *(extra or []), src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def is_stale(src: str = SRC, out: str = LIB) -> bool:
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build())
    sys.exit(0)
