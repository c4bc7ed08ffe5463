"""Builds libw4a16.so in-tree with nvcc for sm_100a.

    python -m weight_only_int4_pack_b200.build [--force] [--debug]

The library is one shared object compiled from csrc/*.cu with the public
header in include/.  --debug builds lib/libw4a16_debug.so instead, with
-DW4_DEBUG: the in-kernel bounds checks of csrc/w4_debug.cuh compiled in
(a failed check sets the device status word and skips its access; the
package loads this library when the environment has W4_DEBUG=1).  The CUDA runtime is linked statically and the driver
API is reached through cudaGetDriverEntryPoint, so the .so loads on a
machine without a GPU (its entry points then fail with W4_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libw4a16.so")
LIB_DEBUG = os.path.join(LIBDIR, "libw4a16_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-Xptxas", "-warn-spills",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def nvcc() -> str:
    for c in ("/usr/local/cuda/bin/nvcc", "nvcc"):
        if os.path.isabs(c) and os.path.exists(c):
            return c
    return "nvcc"


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    objdir = os.path.join(LIBDIR, "obj_debug" if debug else "obj")
    os.makedirs(objdir, exist_ok=True)
    flags = NVCC_FLAGS + (["-DW4_DEBUG"] if debug else [])
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc(), *flags, "-I", INCLUDE, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd))
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    bad = [p.wait() for p in procs]
    if any(bad):
        raise RuntimeError("nvcc failed")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", "-o", tmp, *objs]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
