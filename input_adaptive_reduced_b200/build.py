"""Build librmm.so (the CUDA kernels and the C ABI of include/rmm.h) in-tree
for sm_100a with nvcc.  No torch involvement: the library links the CUDA
runtime statically and hides every symbol except the rmm_* entry points."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librmm.so")
SOURCES = ["rmm_api.cu", "rmm_select.cu", "rmm_pack.cu", "rmm_gemm.cu", "rmm_skinny.cu", "rmm_static.cu",
           "rmm_selftest.cu", "rmm_decode.cu", "rmm_softmax.cu", "rmm_attn.cu",
           "rmm_tiny.cu"]
HEADERS = ["rmm_device.cuh", "rmm_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "rmm.h"))
    files.append(os.path.abspath(__file__))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden",
           "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic",
           "-I", os.path.join(ROOT, "include"),
           "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        cmd += ["-Xptxas", "-v"]
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
