"""Build libdsmoe.so in-tree with nvcc for sm_100a.

    python mixture_experts_layer_score_b200/build.py [--force] [-v] [--role-cycles]

(run by path: importing the package loads the library this script builds)

Each .cu under csrc/ is compiled to an object under _build/ (rebuilt when it or
a header is newer), then linked into mixture_experts_layer_score_b200/libdsmoe.so
with the CUDA runtime linked statically, so the library loads on a host
without a GPU driver (the driver is reached at run time).
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdsmoe.so")
# profiling build with the grouped GEMM's role cycle counters (role_clock.cuh): its own
# objects and library file; load it with DSMOE_LIBRARY=<path> in the environment
ROLE_BUILD = os.path.join(BUILD, "rolecycles")
ROLE_LIB = os.path.join(PKG, "libdsmoe_rolecycles.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def build(force: bool = False, verbose: bool = False, extra_flags=(), role_cycles: bool = False) -> str:
    build_dir, lib = (ROLE_BUILD, ROLE_LIB) if role_cycles else (BUILD, LIB)
    if role_cycles:
        extra_flags = list(extra_flags) + ["-DDSMOE_ROLE_CYCLES"]
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr = _newest_header()
    objs = []
    relinked = force or not os.path.exists(lib)
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr):
            cmd = [nvcc()] + NVCC_FLAGS + list(extra_flags) + ["-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
            relinked = True
    if relinked or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + ".tmp"
        cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", tmp] + objs
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register / smem usage")
    ap.add_argument("--role-cycles", action="store_true",
                    help="profiling build with the grouped GEMM's role cycle counters (libdsmoe_rolecycles.so)")
    args = ap.parse_args()
    extra = ["-Xptxas", "-v"] if args.ptxas_verbose else []
    print(build(force=args.force or args.ptxas_verbose, verbose=args.verbose, extra_flags=extra,
                role_cycles=args.role_cycles))
    sys.exit(0)
