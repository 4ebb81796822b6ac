"""Build ``libh3rr.so`` in-tree with nvcc for sm_100a.

The CUDA runtime is linked statically so the library does not depend on which
libcudart a host process has loaded.  No fast-math, no FMA contraction, no
flush-to-zero: the reduce-scatter's binary32 sums must match the sequential
definition bit for bit.
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libh3rr.so")
DIGEST = LIB + ".sources"  # source_digest() of the build that wrote LIB

NVCC = os.environ.get("NVCC", "nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "--fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC,-Wall,-Wextra,-fvisibility=hidden",
    "--cudart", "static",
    "-Xlinker", "--exclude-libs=ALL",
    "-shared",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def dependencies() -> list[str]:
    """Every file the library is compiled from: sources, internal headers, the
    public header and this script (its flags)."""
    headers = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
    return sources() + sorted(headers) + [os.path.join(INCLUDE, "h3rr.h"), os.path.abspath(__file__)]


def source_digest() -> str:
    """Content digest of dependencies() (file times need not survive a copy)."""
    h = hashlib.sha256()
    for path in dependencies():
        h.update(os.path.relpath(path, ROOT).encode())
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def is_stale() -> bool:
    """True if the library is missing or was built from other sources."""
    if not os.path.exists(LIB) or not os.path.exists(DIGEST):
        return True
    with open(DIGEST) as f:
        return f.read().strip() != source_digest()


def build(verbose: bool = False, extra: list[str] | None = None) -> str:
    cmd = [NVCC, *NVCC_FLAGS, *(extra or []), "-I", INCLUDE, "-I", CSRC, *sources(), "-o", LIB]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    # the digest sits beside the library; extra flags make it a non-default build
    with open(DIGEST, "w") as f:
        f.write(source_digest() if not extra else "custom build\n")
    return LIB


if __name__ == "__main__":
    print(build(verbose=True, extra=sys.argv[1:]))
