"""Build libmoe.so in-tree with nvcc for sm_100a.

    python combine_moe_route_13_b200/build.py [--force] [--verbose] [--ptxas-info] [--check]

--check builds libmoe_check.so instead: the same sources with -DMOE_CHECK_BOUNDS
(every kernel checks its internal index invariants and counts failures, see
moe_debug_bounds_failures in moe.h) and relocatable device code (the failure
counters are one device variable shared by every source file).

(run as a script: importing the package loads the library, which may not
exist yet)

The library is written next to this file so that it travels with the source
tree. Rebuilds only when a source or header is newer than the library.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
LIB_CHECK = os.path.join(HERE, "libmoe_check.so")
SOURCES = ["moe_abi.cu", "route.cu", "dispatch_combine.cu", "gemm_simt.cu", "gemm_tc.cu",
           "route_noalloc.cu", "quant_fp8.cu", "gemm_fp8.cu", "ep.cu"]
HEADERS = [os.path.join(CSRC, h) for h in ("moe_internal.h", "tc_ptx.cuh", "tile_sched.cuh", "fp8_util.cuh",
                                         "vec_util.cuh")] + \
    [os.path.join(ROOT, "include", h) for h in ("moe.h", "moe_ep.h")]
GENCODE = "arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), check: bool = False) -> str:
    lib = LIB_CHECK if check else LIB
    if not force and not needs_build(lib):
        return lib
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    tmp = lib + ".tmp"
    variant = ["-DMOE_CHECK_BOUNDS", "-rdc=true"] if check else []
    cmd = [nvcc_path(), "-shared", "-Xcompiler", "-fPIC", "-O3", "-lineinfo", "-std=c++17",
           "-gencode", GENCODE, *variant, "-I", os.path.join(ROOT, "include"), "-o", tmp, *srcs,
           *extra]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    os.replace(tmp, lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/smem per kernel")
    ap.add_argument("--check", action="store_true", help="build the bounds-checked libmoe_check.so")
    a = ap.parse_args(argv)
    extra = ["-Xptxas", "-v"] if a.ptxas_info else []
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose or a.ptxas_info, extra=extra,
                check=a.check))


if __name__ == "__main__":
    main()
