"""Build the sm_100a shared library ``libsp24.so`` in-tree with nvcc.

Usage: ``python -m structured_sparse_fp8_b200.build`` (or call ``build()``).
The library is a plain C-ABI shared object (see ``include/sp24.h``) with the
CUDA runtime linked statically; it is compiled for sm_100a only.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsp24.so")
SOURCES = ["api.cu", "elementwise.cu", "fp4.cu", "gemm.cu", "int8.cu", "noalloc.cu", "rowscale.cu", "slide.cu", "smallx.cu",
           "stream.cu"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; the sm_100a library cannot be built")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    # every source and header the library is compiled from, whatever its name
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA source into ``libsp24.so`` (skipped when up to date)."""
    if not force and not _stale():
        return LIB
    nvcc = nvcc_path()
    tmp = LIB + ".tmp"
    cmd = [nvcc, "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS,
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC,
           "-Xptxas", "-v" if verbose else "-O3",
           *[os.path.join(CSRC, f) for f in SOURCES], "-o", tmp, "-ldl"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
