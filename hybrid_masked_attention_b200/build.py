"""Build libmtfm.so (the C-ABI CUDA library) in-tree for sm_100a.

    python hybrid_masked_attention_b200/build.py [--force] [--verbose]

Each .cu under csrc/ is compiled to an object in parallel with
``nvcc -gencode arch=compute_100a,code=sm_100a -lineinfo -O3``, then linked
into ``hybrid_masked_attention_b200/libmtfm.so``.  Rebuilds only when a source
or header is newer than the library.

    python hybrid_masked_attention_b200/build.py --debug-bounds

builds the bounds-checked variant (``-DMTFM_DEBUG_BOUNDS``: every TMA coordinate
and computed global row index is tested before use, failures are recorded in the
metadata header) as ``libmtfm_debug_bounds.so`` beside it; the Python binding
loads it instead of libmtfm.so when the environment variable MTFM_LIBRARY names it.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmtfm.so")
DEBUG_BUILD = os.path.join(PKG, "_build_debug_bounds")
DEBUG_LIB = os.path.join(PKG, "libmtfm_debug_bounds.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-I", CSRC, "-I", INCLUDE]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmtfm")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _compile(src: str, verbose: bool, extra, build_dir: str = BUILD) -> str:
    obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    lib, build_dir = (DEBUG_LIB, DEBUG_BUILD) if debug_bounds else (LIB, BUILD)
    if debug_bounds:
        extra = (*extra, "-DMTFM_DEBUG_BOUNDS")
    if not force and up_to_date(lib):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, list(extra), build_dir), sources()))
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill usage")
    ap.add_argument("--debug-bounds", action="store_true", help="build the bounds-checked variant")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug_bounds=a.debug_bounds))
