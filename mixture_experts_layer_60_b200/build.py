"""Builds libmoe.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m mixture_experts_layer_60_b200.build [--verbose] [--ptxas-info] [--check-bounds]

Each csrc/*.cu compiles to an object under _build/ (in parallel), then the
objects link into mixture_experts_layer_60_b200/libmoe.so.  Rebuilds only
what changed (sources or headers newer than the object).  --check-bounds
builds the checked variant instead (-DMOE_CHECK_BOUNDS: internal indices are
tested before each access, failures set a bit of the device error word and
skip the access) into _build_checked/ and libmoe_checked.so; load it by
setting MOE_LIBRARY to its path before importing the package.
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe.so")
BUILD_CHECKED = os.path.join(ROOT, "_build_checked")
LIB_CHECKED = os.path.join(PKG, "libmoe_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(obj: str, deps: list[str]) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False,
          check_bounds: bool = False) -> str:
    bdir, lib_out = (BUILD_CHECKED, LIB_CHECKED) if check_bounds else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                     + glob.glob(os.path.join(ROOT, "include", "*.h")))
    cc = nvcc()
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DMOE_CHECK_BOUNDS"] if check_bounds else [])
    jobs = []
    for src in srcs:
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        if force or ptxas_info or _stale(obj, [src] + headers):
            jobs.append([cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 4)) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or ptxas_info or r.returncode != 0:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {cmd[-3]}")
    objs = [os.path.join(bdir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if jobs or not os.path.exists(lib_out) or _stale(lib_out, objs):
        cmd = [cc, *ARCH, "-shared", "-o", lib_out, *objs, "-lcudart_static", "-lrt", "-ldl",
               "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"link of {os.path.basename(lib_out)} failed")
    return lib_out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--check-bounds", action="store_true")
    a = ap.parse_args()
    print(build(a.verbose, a.ptxas_info, a.force, a.check_bounds))
