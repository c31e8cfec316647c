"""Build libinfllm2.so in-tree for sm_100a with nvcc.

The library is one CUDA translation unit (csrc/infllm2.cu includes the
kernel files).  The CUDA runtime is linked statically and the driver entry
point for tensor maps is looked up at run time, so the library loads on a
machine without a GPU driver (calls then fail with a CUDA error).
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
LIB_PATH = os.path.join(PKG_DIR, "libinfllm2.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def _sources():
    out = [os.path.join(INCLUDE, f) for f in sorted(os.listdir(INCLUDE)) if f.endswith(".h")]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def _nvcc() -> str:
    nv = shutil.which("nvcc")
    if nv:
        return nv
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, out: str = LIB_PATH, defines=()) -> str:
    """Compile csrc/infllm2.cu into libinfllm2.so next to this file (or into
    `out`, with extra -D `defines`)."""
    if out == LIB_PATH and not defines and not force and not needs_build():
        return LIB_PATH
    tmp = out + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, *[f"-D{d}" for d in defines], os.path.join(CSRC, "infllm2.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
