"""Build libmoe_q4.so in-tree with nvcc for sm_100a (no JIT, no torch
extension machinery): ``python -m bit_codebook_quantized_router_b200.build``."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe_q4.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
    "-I" + os.path.join(ROOT, "include"),
]


LIB_DEBUG = os.path.join(PKG, "libmoe_q4_debug.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _build_one(lib, objdir, flags, verbose):
    from concurrent.futures import ThreadPoolExecutor
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    os.makedirs(objdir, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, "-c", src, "-o", obj, *NVCC_FLAGS, *flags]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        return obj

    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc, "-shared", "-o", tmp, *objs, "-gencode", "arch=compute_100a,code=sm_100a",
                           "-Xcompiler", "-fPIC"])
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = True) -> str:
    """Build the release library (and, with debug=True, the bounds-checking
    debug library beside it: MOE_Q4_DEBUG defined)."""
    if force or _stale(LIB):
        _build_one(LIB, os.path.join(PKG, "_build"), list(extra), verbose)
    if debug and (force or _stale(LIB_DEBUG)):
        _build_one(LIB_DEBUG, os.path.join(PKG, "_build_debug"), ["-DMOE_Q4_DEBUG", *extra], verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
