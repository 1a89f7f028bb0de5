"""Build liblsa.so (the C-ABI library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblsa.so")
# the debug build: the same sources with the kernels' bounds checks compiled in
# (-DLSA_BOUNDS_CHECKS=1); a failed check is reported through
# lsa_check_device_errors(), never a trap
LIB_DEBUG = os.path.join(PKG, "liblsa_debug.so")
SOURCES = ["lsa_api.cu", "lsa_build.cu", "lsa_index.cu", "lsa_score_tc.cu", "lsa_attn.cu", "lsa_near_tc.cu",
           "lsa_noalloc.cu", "lsa_shrink.cu", "lsa_shard.cu"]
HEADERS = ["lsa_common.cuh", "lsa_kernels.h", "lsa_tc.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "lsa.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    cmd = [NVCC, *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-I", INCLUDE, "-I", CSRC, "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DLSA_BOUNDS_CHECKS=1"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
