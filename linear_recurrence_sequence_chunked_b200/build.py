"""Build ``libpdn.so`` (the C-ABI CUDA library) in-tree for sm_100a.

Run as ``python -m linear_recurrence_sequence_chunked_b200.build``. Each
``csrc/*.cu`` file is compiled to an object under ``_build/`` (in parallel),
then linked into ``linear_recurrence_sequence_chunked_b200/libpdn.so``.
``--debug-bounds`` builds ``libpdn_debug.so`` instead (objects under
``_build_debug/``): the same sources with PDN_DEBUG_BOUNDS, whose kernels
check their computed indices and record PDN_ERR_BOUNDS in the device error
word rather than access out of range (load it with PDN_LIBRARY=<path>).
"""
from __future__ import annotations

import concurrent.futures
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
LIB = os.path.join(PKG, "libpdn.so")
DEBUG_LIB = os.path.join(PKG, "libpdn_debug.so")
DEBUG_BUILD = os.path.join(ROOT, "_build_debug")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-Wall", "-I", INCLUDE]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpdn.so")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "pdn.h"), __file__])


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, verbose: bool = False, extra_flags=(),
          debug_bounds: bool = False) -> str:
    lib = DEBUG_LIB if debug_bounds else LIB
    bdir = DEBUG_BUILD if debug_bounds else BUILD
    if debug_bounds:
        extra_flags = ["-DPDN_DEBUG_BOUNDS", *extra_flags]
    if not force and not is_stale(lib):
        return lib
    os.makedirs(bdir, exist_ok=True)
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *NVCC_FLAGS, *extra_flags, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed on %s:\n%s%s" % (src, r.stdout, r.stderr))
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [cc, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc link failed:\n%s%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    verbose = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=True, verbose=verbose or bool(extra), extra_flags=extra,
                debug_bounds="--debug-bounds" in sys.argv))
