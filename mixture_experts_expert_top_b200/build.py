"""Build libmoe_b200.so (CUDA C++ for sm_100a) in-tree with nvcc.

The library is plain CUDA: no torch headers, no Python symbols. It links the
CUDA runtime statically and reaches the driver's cuTensorMapEncodeTiled
through the runtime's entry-point query, so it needs only the NVIDIA driver
at run time.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmoe_b200.so")
LIB_DEBUG = os.path.join(HERE, "libmoe_b200_debug.so")
BUILD_DIR = os.path.join(ROOT, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-std=c++17", "-O3", "-lineinfo",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE,
]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + [
        os.path.join(INCLUDE, "moe.h")]


def up_to_date(debug_bounds: bool = False) -> bool:
    lib = LIB_DEBUG if debug_bounds else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug_bounds: bool = False) -> str:
    """Compiles every csrc/*.cu for sm_100a and links the shared library.
    debug_bounds=True builds libmoe_b200_debug.so with -DMOE_DEBUG_BOUNDS
    (range checks on perm-derived row indices and on the expert offsets,
    raising device error 4) from the same sources."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and up_to_date(debug_bounds):
        return lib
    build_dir = os.path.join(BUILD_DIR, "debug_bounds") if debug_bounds else BUILD_DIR
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    flags = NVCC_FLAGS + (["-DMOE_DEBUG_BOUNDS"] if debug_bounds else [])
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *flags, "-c", src, "-o", obj]
        if ptxas_info:
            cmd[1:1] = ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd))
        procs.append((subprocess.Popen(cmd), src))
        objs.append(obj)
    failed = [src for p, src in procs if p.wait() != 0]
    if failed:
        raise RuntimeError(f"nvcc failed on {failed}")
    # The C ABI entry points are exported explicitly; everything else stays hidden.
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           "-Xcompiler", "-fPIC", *objs, "-o", lib + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="-v" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
