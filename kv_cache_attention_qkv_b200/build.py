"""Build libflashcache.so in-tree with nvcc for sm_100a.

    python -m kv_cache_attention_qkv_b200.build [--debug]

Every CUDA/C++ source under ``csrc/`` is compiled into one shared library next
to this file.  The CUDA runtime is linked statically and the driver is reached
through cudaGetDriverEntryPoint, so the library loads on a machine without a
GPU driver (where every call that needs the device returns FC_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libflashcache.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def needs_rebuild() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(PKG, "csrc", "*.h")) + \
        glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, debug: bool = False, verbose: bool = False) -> str:
    if not force and not needs_rebuild():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-std=c++17", "-O3", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", tmp, *sources(), "-ldl", "-lpthread", "-lrt"]
    if debug:
        cmd.insert(1, "-DFC_DEBUG=1")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, debug="--debug" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
