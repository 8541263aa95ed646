"""Builds libspecverify.so in-tree with nvcc for sm_100a (no GPU needed)."""
from __future__ import annotations

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libspecverify.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "specverify.h")])


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile csrc/*.cu into libspecverify.so unless it is newer than every source."""
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = [NVCC, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += sorted(glob.glob(os.path.join(CSRC, "*.cu"))) + ["-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose=True))
