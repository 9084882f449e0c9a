"""Builds the sm_100a shared library ``librmsnorm_b200.so`` in-tree with nvcc.

Usage: ``python residual_add_rmsnorm_rms_b200/build.py [--force] [--verbose-ptxas]``
(run as a file: importing the package itself needs the built library).
nvcc cross-compiles for sm_100a without a GPU. Each source compiles to its own
object (in parallel), then nvcc links the shared library. IEEE division and
square root and no flush-to-zero are spelled out: the kernels rely on them.
The fp8 GEMM unit also needs the CUTLASS/CuTe header tree, which is located
on the Python path (a vendored copy in an installed package).
"""
from __future__ import annotations

import glob
import importlib.util
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librmsnorm_b200.so")
OBJDIR = os.path.join(PKG, "_build")
HEADER = os.path.join(ROOT, "include", "rmsnorm_b200.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [
    *ARCH,
    "-O3", "-lineinfo", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]
# Sources that instantiate CUTLASS templates.
CUTLASS_SOURCES = {"fp8_gemm.cu", "fp8_gemm_ch128.cu", "fp8_gemm_ch64.cu"}
# CUTLASS_ENABLE_GDC_FOR_SM100: the GEMM kernels wait for the previous kernel
# in the stream (griddepcontrol) before touching memory, so they can be
# launched with programmatic dependent launch like the other kernels.
CUTLASS_FLAGS = ["--expt-relaxed-constexpr", "-diag-suppress", "20012",
                 "-DCUTLASS_ENABLE_GDC_FOR_SM100=1"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]


def cutlass_include() -> list[str]:
    """-I flags for a CUTLASS 4 tree with sm100 collectives and tools/util."""
    roots = []
    for pkg, sub in (("flashinfer", ("data", "cutlass")), ("tilelang", ("3rdparty", "cutlass"))):
        spec = importlib.util.find_spec(pkg)
        if spec and spec.submodule_search_locations:
            roots.append(os.path.join(list(spec.submodule_search_locations)[0], *sub))
    for r in roots:
        inc, util = os.path.join(r, "include"), os.path.join(r, "tools", "util", "include")
        if (os.path.exists(os.path.join(inc, "cutlass", "gemm", "collective", "builders",
                                        "sm100_umma_builder.inl"))
                and os.path.exists(os.path.join(util, "cutlass", "util", "packed_stride.hpp"))):
            return ["-I" + inc, "-I" + util]
    raise RuntimeError("no CUTLASS 4 header tree with sm100 support found on the Python path")


def _deps(path: str, seen: set | None = None) -> set:
    """`path` and every repository header it includes, transitively."""
    seen = set() if seen is None else seen
    if path in seen or not os.path.exists(path):
        return seen
    seen.add(path)
    with open(path, errors="replace") as f:
        for line in f:
            line = line.strip()
            if line.startswith("#include") and '"' in line:
                inc = line.split('"')[1]
                _deps(os.path.normpath(os.path.join(os.path.dirname(path), inc)), seen)
    return seen


def _obj(src: str) -> str:
    return os.path.join(OBJDIR, os.path.basename(src) + ".o")


def _obj_stale(src: str) -> bool:
    obj = _obj(src)
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in _deps(src) | {__file__})


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in sources() + headers() + [__file__])


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")


def _compile(src: str, verbose_ptxas: bool, force: bool = True) -> str:
    name = os.path.basename(src)
    obj = _obj(src)
    if not force and not _obj_stale(src):
        return obj
    cmd = [nvcc(), *NVCC_FLAGS]
    if name in CUTLASS_SOURCES:
        cmd += CUTLASS_FLAGS + cutlass_include()
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-c", src, "-o", obj]
    subprocess.check_call(cmd)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    srcs = sources()
    # Objects are rebuilt when their source or an included header changed
    # (all of them with force or verbose_ptxas).
    every = force or verbose_ptxas
    with ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, every), srcs))
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), *ARCH, "-shared", *objs, "-o", tmp, "-lcuda"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
