"""Build liblh.so (sm_100a) in-tree with nvcc.

Usage: ``python -m long_context_symmetric_b200.build`` (or ``build()`` from
Python). Objects go to ``_build/`` at the repository root; the shared library
lands next to this file so that it travels with the source tree.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "liblh.so")
# debug build: device-side bounds checks on the indices read from the map and
# slot table (-DLH_DEBUG_BOUNDS), objects and library kept apart
DEBUG_OBJDIR = os.path.join(OBJDIR, "debug_bounds")
DEBUG_LIB = os.path.join(PKG, "liblh_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(DEBUG_OBJDIR if debug else OBJDIR, os.path.basename(src) + ".o")
    deps = [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "lh.h")]
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(d) for d in deps):
        return obj
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DLH_DEBUG_BOUNDS"] if debug else []), "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile every CUDA source for sm_100a and link liblh.so (liblh_debug.so
    with the device-side bounds checks); returns its path."""
    objdir, lib = (DEBUG_OBJDIR, DEBUG_LIB) if debug_bounds else (OBJDIR, LIB)
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug_bounds), srcs))
    if os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(o) for o in objs):
        return lib
    cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
