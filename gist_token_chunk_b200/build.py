"""Build step for libssa.so (sm_100a) -- run by ``__graft_entry__.build()``.

Compiles the CUDA kernels and the C ABI with nvcc into
``gist_token_chunk_b200/libssa.so`` (in-tree, static CUDA runtime).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libssa.so")
SOURCES = ["ssa_kernels.cu", "ssa_api.cpp", "ssa_prefill.cu"]
HEADERS = ["ssa_device.cuh", "ssa_fused.cuh", "ssa_generic.cuh", "ssa_internal.h", "ssa_pipe.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "ssa.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    """Compile libssa.so; ``extra`` nvcc flags (e.g. -DSSA_TRACE) and another
    ``out`` path give instrumented variants without touching the product."""
    if out == LIB and not force and not _stale():
        return LIB
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *[os.path.join(CSRC, f) for f in SOURCES], *extra]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
