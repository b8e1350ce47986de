"""Build the KDA CUDA library (libkda.so) in-tree for sm_100a.

The library is one translation unit (csrc/kda_api.cu includes the kernels)
compiled with nvcc for compute_100a / sm_100a and linked as a shared object
next to this file.  No JIT cache is involved, so the built file travels with
the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkda.so")
LIB_PHASE = os.path.join(HERE, "libkda_phase.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "kda.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, phase_clocks: bool = False) -> str:
    """Builds libkda.so (or, with phase_clocks, the instrumented libkda_phase.so
    that accumulates per-phase cycle counts of the fused kernel)."""
    lib = LIB_PHASE if phase_clocks else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"),
           os.path.join(CSRC, "kda_api.cu"), "-o", tmp, "-lcuda"]
    if phase_clocks:
        cmd.insert(1, "-DKDA_PHASE_CLOCKS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                phase_clocks="--phase-clocks" in sys.argv))
