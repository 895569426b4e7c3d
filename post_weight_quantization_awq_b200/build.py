"""Builds libawq.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m post_weight_quantization_awq_b200.build [--force] [--verbose] [--debug-bounds]

Each .cu under csrc/ is compiled to an object under _build/ (rebuilt when it
or a header is newer), then linked into post_weight_quantization_awq_b200/libawq.so
with the CUDA runtime linked statically.  --debug-bounds builds the debug
library libawq_debug.so instead (objects under _build/debug/, compiled with
-DAWQ_DEBUG_BOUNDS: index checks in the kernels, read by awq_bounds_status;
the binding loads it when AWQ_LIB=debug).  No GPU is needed to build.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libawq.so")
DEBUG_LIB = os.path.join(PKG, "libawq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
                     "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug_bounds: bool = False) -> str:
    nvcc = _nvcc()
    build_dir = os.path.join(BUILD_DIR, "debug") if debug_bounds else BUILD_DIR
    lib = DEBUG_LIB if debug_bounds else LIB
    if debug_bounds:
        extra_flags = (*extra_flags, "-DAWQ_DEBUG_BOUNDS")
    os.makedirs(build_dir, exist_ok=True)
    headers = _headers()
    objs = []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(lib, objs):
        tmp = lib + ".tmp"
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true", help="print register / smem usage")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build libawq_debug.so with index checks in the kernels")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_v else []
    print(build(force=a.force or a.ptxas_v, verbose=a.verbose, extra_flags=extra,
                debug_bounds=a.debug_bounds))
    return 0


if __name__ == "__main__":
    sys.exit(main())
