"""Build the CUDA library (libqlora.so) in-tree with nvcc for sm_100a.

The library is a plain C ABI (include/qlora.h) with the CUDA runtime linked statically, so the
shared object loads on a machine without a GPU driver (entry points then report QLORA_ERR_CUDA on
their first CUDA call) and carries no dependency on PyTorch.

build(debug=True) compiles the same sources with -DQLORA_DEBUG into libqlora_debug.so: the kernels
then check their own index arithmetic (TMA start coordinates, partial-sum pieces and segments,
arrival counters, output rows) before each access it computes, and record QLORA_ERR_INVALID_ARG
in the status word instead of touching memory out of range.  The binding loads it when the
environment sets QLORA_LIBRARY=debug.
"""
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqlora.so")
LIB_DEBUG = os.path.join(PKG, "libqlora_debug.so")
SOURCES = ["qlora.cu"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(INCLUDE, "qlora.h")]
    for f in os.listdir(CSRC):
        if f.endswith((".cu", ".cuh", ".h")):
            files.append(os.path.join(CSRC, f))
    return files


def up_to_date(lib=LIB):
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force=False, verbose=False, extra_flags=(), debug=False):
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
           "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-I", CSRC, "-Xptxas", "-v" if verbose else "-O3",
           *(["-DQLORA_DEBUG"] if debug else []), *extra_flags,
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
