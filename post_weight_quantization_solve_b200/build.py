"""Build libgptq.so in-tree for sm_100a with nvcc (no JIT, no torch extension).

    python -m post_weight_quantization_solve_b200.build [--force] [-v]
"""
from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgptq.so")
# the index-checking variant (GPTQ_DEBUG_BOUNDS: record-and-skip checks in the kernels)
OUT_DBG = os.path.join(PKG, "_build_dbg")
LIB_DBG = os.path.join(PKG, "libgptq_dbg.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
         "-I", CSRC, "--expt-relaxed-constexpr"]


def _newer(src, dst, deps):
    if not os.path.exists(dst):
        return True
    t = os.path.getmtime(dst)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


def build(force=False, verbose=False, extra=(), debug_bounds=False):
    """Compile every translation unit and link the library; returns its path. With
    debug_bounds, the index-checking variant libgptq_dbg.so (objects in _build_dbg)."""
    out, lib = (OUT_DBG, LIB_DBG) if debug_bounds else (OUT, LIB)
    if debug_bounds:
        extra = (*extra, "-DGPTQ_DEBUG_BOUNDS")
    os.makedirs(out, exist_ok=True)
    headers = (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
               glob.glob(os.path.join(ROOT, "include", "*.h")))
    objs, cmds = [], []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(out, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _newer(src, obj, headers):
            cmds.append([NVCC, *FLAGS, *extra, "-c", src, "-o", obj])
    # the translation units compile independently: one nvcc per file, several at a time
    # (the longest file sets the build time)
    def compile_one(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        return subprocess.run(cmd, capture_output=not verbose, text=True)
    workers = max(1, min(len(cmds), os.cpu_count() or 1, 8))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
        results = list(pool.map(compile_one, cmds))
    for cmd, r in zip(cmds, results):
        if r.returncode != 0:
            if not verbose:
                sys.stderr.write(r.stdout + r.stderr)
            raise subprocess.CalledProcessError(r.returncode, cmd)
        if not verbose and r.stderr.strip():
            sys.stderr.write(r.stderr)
    if force or any(_newer(o, lib, []) for o in objs):
        cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", lib]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build the index-checking variant libgptq_dbg.so")
    a = ap.parse_args()
    build(a.force, a.v, ("-Xptxas", "-v") if a.ptxas_v else (), debug_bounds=a.debug_bounds)
    sys.exit(0)
