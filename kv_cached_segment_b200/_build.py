"""Builds libnomas.so in-tree with nvcc for sm_100a.

Usage: ``python -m kv_cached_segment_b200._build [-v]``.  The library links
the CUDA runtime statically and reaches the driver API only through the
runtime's entry-point query, so it loads on machines without a GPU driver.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libnomas.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = ["abi.cu", "rope_append.cu", "select.cu", "attention.cu", "attention_pair.cu", "frame_picker.cu", "merge.cu",
           "noalloc.cu"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O3",
              "--expt-relaxed-constexpr", "-cudart", "static"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "nomas.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    """Compiles every source and links libnomas.so; returns its path."""
    if not force and not _stale():
        return LIB_PATH
    nvcc = nvcc_path()
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc, *ARCH_FLAGS, *NVCC_FLAGS, "-shared", "-I", INCLUDE, "-I", CSRC,
           *(os.path.join(CSRC, s) for s in SOURCES), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
