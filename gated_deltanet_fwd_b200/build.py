"""Builds libgdn.so in-tree with nvcc for sm_100a (cross-compiles on a host without a GPU).

    python -m gated_deltanet_fwd_b200.build [--force] [--verbose]

Each csrc/*.cu is compiled to an object under _build/ (rebuilt when it or a header is newer),
then all are linked into gated_deltanet_fwd_b200/libgdn.so with the CUDA runtime linked
statically and libcuda resolved at run time (no driver library needed at link time).

A second library, libgdn_debug.so (objects under _build_debug/), is the same code built for the
failure tests only: every bounded device wait gives up after about a millisecond instead of
seconds, and an extra export (gdn_debug_set_skip_chunk) makes the tensor-core prefill withhold
one chunk's tiles so that those waits run out.  The product path never loads it.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgdn.so")
DEBUG_BUILD = os.path.join(PKG, "_build_debug")
DEBUG_LIB = os.path.join(PKG, "libgdn_debug.so")
DEBUG_FLAGS = ["-DGDN_DEBUG_WAIT_NS=1000000ull", "-DGDN_FAULT_INJECTION"]
INCLUDE = os.path.join(ROOT, "include")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          debug: bool = False) -> str:
    """Builds libgdn.so (or, with debug=True, the failure-test library libgdn_debug.so)."""
    build_dir, lib_path = (DEBUG_BUILD, DEBUG_LIB) if debug else (BUILD, LIB)
    extra = DEBUG_FLAGS if debug else []
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_hdr = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    objs = []
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_hdr)):
            continue
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
    if (force or not os.path.exists(lib_path)
            or os.path.getmtime(lib_path) < max(os.path.getmtime(o) for o in objs)):
        tmp = lib_path + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    for dbg in (False, True):
        print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                    ptxas_verbose="--ptxas" in sys.argv, debug=dbg))
