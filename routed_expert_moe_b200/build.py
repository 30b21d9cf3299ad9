"""Build the sm_100a shared library in-tree (nvcc; no JIT cache).

    python routed_expert_moe_b200/build.py [--force] [-v]

Each ``csrc/*.cu`` is compiled to an object for ``sm_100a`` and the objects
are linked into ``_lib/libmoe_b200.so`` with the CUDA runtime linked
statically, so the library only needs the driver at run time.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
OUT_DIR = PKG / "_lib"
LIB = OUT_DIR / "libmoe_b200.so"
INCLUDE = PKG.parent / "include"

NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", str(INCLUDE)]


def sources():
    return sorted(CSRC.glob("*.cu"))


def _deps():
    return sources() + sorted(CSRC.glob("*.cuh")) + [INCLUDE / "moe.h"]


def stale() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(p.stat().st_mtime > t for p in _deps())


def _compile(src: Path, verbose_ptxas: bool) -> Path:
    obj = OUT_DIR / (src.stem + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, "-c", str(src), "-o", str(obj)]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> Path:
    if not force and not stale():
        return LIB
    OUT_DIR.mkdir(parents=True, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas), sources()))
    tmp = LIB.with_suffix(".so.tmp")
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", str(tmp), *map(str, objs)])
    os.replace(tmp, LIB)
    for o in objs:
        o.unlink()
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
