"""Build of the native library libsitu_glu.so (nvcc, sm_100a, in-tree).

nvcc cross-compiles for sm_100a without a GPU, so this runs anywhere the CUDA
toolkit is installed.  The shared object is written next to this file so that
it travels with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
SOURCES = [os.path.join(PKG_DIR, "csrc", "situ_glu.cu")]
HEADERS = [os.path.join(ROOT, "include", "situ_glu.h"), os.path.join(PKG_DIR, "csrc", "situ_fused_gemm.cuh")]
LIBRARY = os.path.join(PKG_DIR, "libsitu_glu.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put the CUDA toolkit on PATH")


def is_stale(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return True
    t = os.path.getmtime(output)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build_library(force: bool = False, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile the CUDA sources into ``output`` unless it is up to date."""
    if not force and not is_stale(output):
        return output
    tmp = output + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-I", os.path.join(ROOT, "include"),
           *SOURCES, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


if __name__ == "__main__":
    print(build_library(force=True))
