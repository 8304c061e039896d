"""Build libpa.so in-tree: nvcc for sm_100a (device code) + the host C++ sources.

    python paged_kv_cache_428_b200/build.py [--verbose-ptxas]

The .so lands next to this file, where the Python binding loads it from.  This script
imports nothing from the package, so it runs before the library exists.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libpa.so"
SOURCES = [CSRC / "pa_lib.cu", CSRC / "host.cpp", CSRC / "allocator.cpp"]
HEADERS = [ROOT / "include" / "pa.h", CSRC / "common.cuh", CSRC / "cache_ops.cuh", CSRC / "decode.cuh", CSRC / "decode_mma.cuh", CSRC / "decode_balanced.cuh", CSRC / "decode_allheads.cuh", CSRC / "decode_q8.cuh", CSRC / "prefill.cuh", CSRC / "prefill_tc.cuh", CSRC / "tc.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(p.stat().st_mtime > t for p in SOURCES + HEADERS)


def build(verbose_ptxas: bool = False, force: bool = False) -> Path:
    if not force and not stale():
        return LIB
    cmd = [nvcc(), *NVCC_FLAGS, "-I", str(ROOT / "include"), "-I", str(CSRC)]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [str(s) for s in SOURCES] + ["-o", str(LIB)]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True)
    print(LIB)
