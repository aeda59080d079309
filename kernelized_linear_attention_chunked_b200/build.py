"""Build libkata.so in-tree for sm_100a with nvcc.

Each .cu file under csrc/ is compiled to an object in _build/ (in parallel),
then linked into kernelized_linear_attention_chunked_b200/libkata.so with the
static CUDA runtime. Only the extern "C" entry points of include/kata.h are
exported. build(debug=True) compiles the same sources with -DKATA_DEBUG (the
device-side bounds checks) into _build_debug/ and libkata_debug.so.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
BUILD = ROOT / "_build"
LIB = PKG / "libkata.so"
BUILD_DEBUG = ROOT / "_build_debug"
LIB_DEBUG = PKG / "libkata_debug.so"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", str(ROOT / "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and Path(cand).exists():
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu"))


def _compile(src: Path, extra: list[str], build_dir: Path) -> Path:
    obj = build_dir / (src.stem + ".o")
    deps = [src] + list(CSRC.glob("*.cuh")) + list(CSRC.glob("*.h")) + [ROOT / "include" / "kata.h"]
    if obj.exists() and obj.stat().st_mtime > max(p.stat().st_mtime for p in deps):
        return obj
    cmd = [nvcc()] + NVCC_FLAGS + extra + ["-c", str(src), "-o", str(obj)]
    subprocess.run(cmd, check=True)
    return obj


def build(verbose_ptxas: bool = False, debug: bool = False) -> Path:
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    build_dir.mkdir(exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DKATA_DEBUG"] if debug else [])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, build_dir), sources()))
    tmp = lib.with_suffix(".so.tmp")
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", str(tmp)] + [str(o) for o in objs]
    subprocess.run(cmd, check=True)
    tmp.replace(lib)
    return lib


if __name__ == "__main__":
    import sys
    print(build(verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))
