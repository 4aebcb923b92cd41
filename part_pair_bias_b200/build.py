"""Build step of the CUDA library: nvcc, sm_100a, in-tree shared object."""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(_HERE)
SRC = os.path.join(_HERE, "csrc", "pairbias.cu")
CSRC = os.path.join(_HERE, "csrc")
# every source the library is compiled from (pairbias.cu includes the rest)
DEPS = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))) + [
    os.path.join(ROOT, "include", "pairbias.h")]
OUT = os.path.join(_HERE, "libpairbias.so")
# the same library with every computed-index check of PB_DEBUG_BOUNDS compiled in
OUT_DEBUG = os.path.join(_HERE, "libpairbias_debug.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile libpairbias.so (or, with debug, libpairbias_debug.so) if it is
    missing or older than a source file."""
    out = OUT_DEBUG if debug else OUT
    stale = force or not os.path.exists(out) or any(os.path.getmtime(d) > os.path.getmtime(out) for d in DEPS)
    if stale:
        nvcc = os.environ.get("NVCC", "nvcc")
        cmd = [nvcc, *NVCC_FLAGS, *(["-DPB_DEBUG_BOUNDS"] if debug else []), "-I", os.path.join(ROOT, "include"),
               "-o", out + ".tmp", SRC]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose=True))
