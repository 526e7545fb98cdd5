"""In-tree builds of the package's native libraries.

* ``libta23.so``        - the CUDA library behind the C ABI in ``include/ta23.h``
                          (sm_100a only: nvcc -gencode arch=compute_100a,code=sm_100a).
* ``libta23_synth.so``  - the seeded input generator (plain C).

Each library is rebuilt when it is missing or older than any of its sources.
Builds are atomic (compile to a temporary file, then rename), so concurrent
test processes never load a half-written library.
"""
from __future__ import annotations

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

LIB_CUDA = os.path.join(PKG, "libta23.so")
LIB_SYNTH = os.path.join(PKG, "libta23_synth.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def cuda_sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def cuda_deps() -> list[str]:
    return (cuda_sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + sorted(glob.glob(os.path.join(INCLUDE, "*.h"))))


def build_cuda(force: bool = False, verbose: bool = False) -> str:
    """Compile every ``csrc/*.cu`` into ``libta23.so`` for sm_100a."""
    if force or _stale(LIB_CUDA, cuda_deps()):
        tmp = LIB_CUDA + f".tmp{os.getpid()}"
        cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *cuda_sources()]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        os.replace(tmp, LIB_CUDA)
    return LIB_CUDA


def build_synth(force: bool = False) -> str:
    """Compile the seeded input generator into ``libta23_synth.so``."""
    src = os.path.join(CSRC, "synthetic.c")
    if force or _stale(LIB_SYNTH, [src]):
        tmp = LIB_SYNTH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, LIB_SYNTH)
    return LIB_SYNTH


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_cuda(force)
