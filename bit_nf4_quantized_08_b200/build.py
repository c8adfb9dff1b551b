"""Build the in-tree CUDA library ``libqlora_nf4.so`` for sm_100a.

The library is one translation unit (``csrc/qlora_nf4.cu``) compiled with
nvcc into a shared object that exports the C ABI of ``include/qlora_nf4.h``.
The CUDA runtime is linked statically, so the library loads (and its host-side
argument checks run) on machines without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "qlora_nf4.cu")
LIB = os.path.join(HERE, "libqlora_nf4.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _sources() -> list[str]:
    out = [os.path.join(HERE, "..", "include", "qlora_nf4.h")]
    for name in sorted(os.listdir(SRC_DIR)):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(SRC_DIR, name))
    return out


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
