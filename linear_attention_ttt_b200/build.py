"""Builds libttt_b200.so in-tree from csrc/*.cu for sm_100a with nvcc.

    python -m linear_attention_ttt_b200.build [--force] [--verbose] [--debug-bounds]

--debug-bounds builds libttt_b200_dbg.so instead (objects under csrc/_build_dbg/),
compiled with -DTTT_DEBUG_BOUNDS: the kernels check their index arithmetic
and report a failed check as TTT_ERR_BOUNDS through ttt_get_device_status.

Each translation unit is compiled to an object under csrc/_build/ and the
objects are linked into linear_attention_ttt_b200/libttt_b200.so (cudart
linked statically, so the library shares the CUDA driver context of whatever
process loads it). A unit is rebuilt when it, or any header it may include,
is newer than its object.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(CSRC, "_build")
LIB = os.path.join(PKG, "libttt_b200.so")
BUILD_DBG = os.path.join(CSRC, "_build_dbg")
LIB_DBG = os.path.join(PKG, "libttt_b200_dbg.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    build_dir, lib = (BUILD_DBG, LIB_DBG) if debug_bounds else (BUILD, LIB)
    if debug_bounds:
        extra = (*extra, "-DTTT_DEBUG_BOUNDS")
    os.makedirs(build_dir, exist_ok=True)
    hdr_time = max([os.path.getmtime(h) for h in _headers()] + [0])
    objs = []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_time)):
            continue
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0 or verbose:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}")
    newest = max(os.path.getmtime(o) for o in objs)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < newest:
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", lib, "-lcuda"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, debug_bounds=args.debug_bounds))
