"""Build libmq.so (the CUDA kernels and the C ABI) in-tree with nvcc for sm_100a,
and libmq_debug.so, the same sources with the bounds checks of MQ_DEBUG.

Usage: python -m nvfp4_w4a4_quantized_03_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmq.so")
DEBUG_LIB = os.path.join(HERE, "libmq_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps.append(os.path.join(HERE, "..", "include", "mq.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _build_one(lib: str, objdir: str, extra, ptxas_verbose: bool) -> None:
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
                    "-I", os.path.join(HERE, "..", "include")] + list(extra)
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        subprocess.check_call([nvcc(), "-c", src, "-o", obj] + flags)
        objs.append(obj)
    tmp = lib + ".tmp"
    subprocess.check_call([nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-lcudart_static"])
    os.replace(tmp, lib)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Build both libraries if a source is newer (or `force`); returns libmq.so's path."""
    if force or _stale(LIB):
        _build_one(LIB, os.path.join(HERE, "_build"), [], ptxas_verbose)
    if force or _stale(DEBUG_LIB):
        _build_one(DEBUG_LIB, os.path.join(HERE, "_build", "debug"), ["-DMQ_DEBUG=1"], ptxas_verbose)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
