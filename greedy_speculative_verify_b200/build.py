"""Builds libvgv.so in-tree with nvcc for sm_100a.

``python -m greedy_speculative_verify_b200.build`` (or ``build()``) compiles
``csrc/vgv_api.cu`` (which includes every kernel header) into
``greedy_speculative_verify_b200/libvgv.so``. The build is skipped when the
library is newer than every source and header.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libvgv.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    # the router's fp32 chain must round exactly as written
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


DEBUG_LIB = os.path.join(PKG, "libvgv_debug.so")


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None, out: str | None = None) -> str:
    """Builds the library (out=None: LIB, skipped when up to date). out names
    another file, e.g. DEBUG_LIB with extra_flags=["-DVG_DEBUG_BOUNDS"]."""
    target = out or LIB
    if not force and (up_to_date() if out is None else
                      os.path.exists(target) and all(os.path.getmtime(s) <= os.path.getmtime(target) for s in sources())):
        return target
    tmp = target + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "vgv_api.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout, r.stderr, sep="\n")
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
