"""Builds the CUDA library ``libpagedkv.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m paged_kv_cache_344_b200.build [--force]``.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpagedkv.so")
MAIN = os.path.join(CSRC, "pagedkv.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    files = [os.path.join(INCLUDE, "pagedkv.h")]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            files.append(os.path.join(CSRC, name))
    return files


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in sources())


def build_library(force: bool = False, extra_flags: list[str] | None = None, out: str = LIB,
                  verbose: bool = False) -> str:
    """Compile ``csrc/pagedkv.cu`` into ``out`` unless it is up to date."""
    if not force and not is_stale(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC, MAIN, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build_library(force=force or bool(extra), extra_flags=extra, verbose=True))
