"""Build libpagedkv.so (the CUDA library behind include/pagedkv.h) for sm_100a.

``python -m paged_kv_cache_386_b200.build`` compiles in place with nvcc; the
library links the CUDA runtime statically, so it loads without a GPU.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libpagedkv.so"
SOURCES = [CSRC / "pkv_api.cu", CSRC / "pkv_block_manager.cpp"]
HEADERS = sorted(CSRC.glob("*.cuh")) + [ROOT / "include" / "pagedkv.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def command(out: Path = LIB, verbose_ptxas: bool = False) -> list[str]:
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", "-I", str(ROOT / "include"), "-I", str(CSRC),
           "-Xcompiler", "-Wall", "--expt-relaxed-constexpr"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    return cmd + ["-o", str(out), *map(str, SOURCES)]


def stale(out: Path = LIB) -> bool:
    if not out.exists():
        return True
    t = out.stat().st_mtime
    return any(p.stat().st_mtime > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose_ptxas: bool = False) -> Path:
    if force or stale():
        subprocess.run(command(verbose_ptxas=verbose_ptxas), check=True)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="-v" in sys.argv)
    print(LIB)
