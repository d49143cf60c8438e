"""Build the JetBlock CUDA library (libjet.so) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libjet.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    out = []
    for d, _, files in os.walk(CSRC):
        out += [os.path.join(d, f) for f in files if f.endswith((".cu", ".cuh", ".h"))]
    out.append(os.path.join(INCLUDE, "jet.h"))
    return out


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, out: str = LIB) -> str:
    """Compile csrc/jet_api.cu (which includes every kernel) into libjet.so
    (or, for a test build with extra defines, into `out`)."""
    if not force and os.path.exists(out):
        mt = os.path.getmtime(out)
        if all(os.path.getmtime(s) <= mt for s in sources()):
            return out
    cmd = [NVCC, *FLAGS, *(extra or []), "-I", INCLUDE, "-I", CSRC,
           "-o", out + ".tmp", os.path.join(CSRC, "jet_api.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
