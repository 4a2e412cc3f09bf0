"""Build librlscan.so (sm_100a) in-tree with nvcc.

One translation unit (csrc/rlscan_api.cu) holds the host entry points and
every kernel instantiation; the CUDA runtime is linked statically so the
library only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "librlscan.so")
SOURCES = [os.path.join(CSRC, "rlscan_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "rlscan.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "--expt-relaxed-constexpr",
    "-shared", "-cudart", "static",
]


def source_hash() -> str:
    """Hash of every kernel source (csrc/) and the build flags: identifies the
    kernels a profile was taken on (the public header's comments do not)."""
    h = hashlib.sha256()
    for path in sorted(d for d in DEPS if os.path.dirname(d) == CSRC):
        h.update(os.path.basename(path).encode())
        with open(path, "rb") as f:
            h.update(f.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()[:16]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and os.path.exists(OUT):
        t = os.path.getmtime(OUT)
        if all(os.path.getmtime(d) <= t for d in DEPS):
            return OUT
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose_ptxas else []),
           "-I", os.path.join(ROOT, "include"), *SOURCES, "-o", OUT + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
