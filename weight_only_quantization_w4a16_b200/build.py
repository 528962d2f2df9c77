"""Builds libawq_w4a16.so in-tree with nvcc for sm_100a.

    python -m weight_only_quantization_w4a16_b200.build [--force]
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
LIB_NAME = "libawq_w4a16.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
# the same library with the kernels' index checks compiled in (-DAWQ_DEBUG_BOUNDS): a failed check
# is reported by awq_poll_device_status as AWQ_ERR_BOUNDS instead of touching memory out of bounds
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libawq_w4a16_debug_bounds.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def _sources():
    out = []
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".map")):
            out.append(os.path.join(CSRC, f))
    out.append(os.path.join(INCLUDE, "awq_w4a16.h"))
    return out


def needs_build(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in _sources())


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libawq_w4a16")
    return cand


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug_bounds: bool = False) -> str:
    """Compiles the library (or its bounds-checking debug variant) if a source is newer."""
    out = DEBUG_LIB_PATH if debug_bounds else LIB_PATH
    if debug_bounds:
        extra_flags = (*extra_flags, "-DAWQ_DEBUG_BOUNDS")
    if not force and not needs_build(out):
        return out
    tmp = out + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra_flags,
           "-I", INCLUDE, "-I", CSRC,
           "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
           os.path.join(CSRC, "awq_lib.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, flush=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [],
          debug_bounds="--debug-bounds" in sys.argv)
