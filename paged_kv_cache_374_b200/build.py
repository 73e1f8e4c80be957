"""Build libpa.so, the C-ABI library, in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_374_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBRARY = os.path.join(PKG, "libpa.so")
SOURCES = ["allocator.cpp", "reshape_and_cache.cu", "paged_decode.cu", "paged_decode_noalloc.cu", "copy_blocks.cu",
           "paged_prefill.cu", "selftest.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC,-O2,-Wall", "-shared", "-cudart", "static"]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return files


def needs_build() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIBRARY
    nvcc = os.environ.get("NVCC") or ("nvcc" if _on_path("nvcc") else "/usr/local/cuda/bin/nvcc")
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


def _on_path(exe: str) -> bool:
    return any(os.access(os.path.join(d, exe), os.X_OK) for d in os.environ.get("PATH", "").split(os.pathsep))


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
