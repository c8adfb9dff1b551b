"""Build the in-tree CUDA library ``libqlora_nf4.so`` for sm_100a.

The library is one translation unit (``csrc/qlora_nf4.cu``) compiled with
nvcc into a shared object that exports the C ABI of ``include/qlora_nf4.h``.
The CUDA runtime is linked statically, so the library loads (and its host-side
argument checks run) on machines without a GPU.

``build(debug=True)`` compiles the same sources with ``-DQLORA_DEBUG`` into
``libqlora_nf4_debug.so``: device-side bounds checks of the computed store
indices, each of which records QLORA_ERR_BOUNDS in the status word and
skips the store instead of trapping.  The binding loads it when the
environment variable QLORA_LIBRARY is "debug".
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "qlora_nf4.cu")
LIB = os.path.join(HERE, "libqlora_nf4.so")
LIB_DEBUG = os.path.join(HERE, "libqlora_nf4_debug.so")

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


def needs_build(debug: bool = False) -> bool:
    lib = LIB_DEBUG if debug else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _sources())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(debug):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc, *NVCC_FLAGS, *(["-DQLORA_DEBUG"] if debug else []), "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
