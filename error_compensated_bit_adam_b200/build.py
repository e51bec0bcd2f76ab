"""Build libonebit.so in-tree with nvcc for sm_100a (B200).

    python -m error_compensated_bit_adam_b200.build [--verbose-ptxas]

The library is a plain C-ABI shared object (no torch types); the Python
binding loads it with ctypes.  CUDA's runtime is linked statically.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, "onebit.cu")]
DEPENDS = SOURCES + [os.path.join(CSRC, "onebit_kernels.cuh"), os.path.join(ROOT, "include", "onebit.h")] + [
    os.path.join(CSRC, "kernels", f) for f in sorted(os.listdir(os.path.join(CSRC, "kernels")))]
LIBRARY = os.path.join(HERE, "libonebit.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "-shared",
    "-Xcompiler", "-fPIC,-fvisibility=hidden,-Wall",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libonebit")


def stale() -> bool:
    if not os.path.exists(LIBRARY):
        return True
    t = os.path.getmtime(LIBRARY)
    return any(os.path.getmtime(p) > t for p in DEPENDS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIBRARY
    tmp = LIBRARY + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose_ptxas else []), "-o", tmp, *SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv))
