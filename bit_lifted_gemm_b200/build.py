"""Build liblq.so (the C-ABI library of sm_100a kernels) in-tree with nvcc.

    python bit_lifted_gemm_b200/build.py [--force] [--verbose-ptxas] [--debug]

--debug builds liblq_debug.so instead: the same sources with -DLQ_DEBUG, whose
kernels check the element index of each computed global access against its
buffer and report LQ_ERR_BOUNDS instead of touching memory out of bounds. The
package loads it when the environment has LQ_DEBUG=1.
(Run it by path: importing the package loads the library.)
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
LIB = os.path.join(PKG, "liblq.so")
OBJDIR = os.path.join(PKG, "_build")
LIB_DEBUG = os.path.join(PKG, "liblq_debug.so")
OBJDIR_DEBUG = os.path.join(PKG, "_build_debug")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    objdir, lib = (OBJDIR_DEBUG, LIB_DEBUG) if debug else (OBJDIR, LIB)
    flags = FLAGS + (["-DLQ_DEBUG"] if debug else [])
    os.makedirs(objdir, exist_ok=True)
    headers = _headers()
    objs = []
    for src in _sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or ptxas_verbose or _stale(obj, [src] + headers):
            cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            subprocess.check_call(cmd)
    if force or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt",
                               "-lpthread"])
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv,
                debug="--debug" in sys.argv))
