"""Build the in-tree C-ABI library ``libpod_attn.so`` (sm_100a) with nvcc.

The library is self-contained: the CUDA runtime is linked statically and the
driver entry point for tensor-map encoding is looked up at run time, so the
.so loads on a machine without a GPU (plan/ABI tests) and carries no JIT cache.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpod_attn.so")
SOURCES = [os.path.join(CSRC, f) for f in ("pod_attn.cu", "plan.cpp", "pod_static.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("pod_plan.h", "pod_ptx.cuh")] + [os.path.join(INCLUDE, "pod_attn.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libpod_attn.so if it is missing or older than its sources."""
    if not force and not _stale():
        return LIB
    cmd = [NVCC, "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-cudart", "static", "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
