"""Build the package's native libraries in-tree.

* ``synth/libtre_synth.so`` — the seeded input generator (gcc + OpenMP).
* ``libtre.so``             — the engine: host planner + C ABI (C++17) and the
                              persistent sm_100a kernel (nvcc, -gencode
                              arch=compute_100a,code=sm_100a).

Run ``python -m persistent_tile_pipelined_b200.build``.  nvcc cross-compiles without a
GPU, so this works on a CPU-only machine.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
ENGINE_LIB = os.path.join(PKG, "libtre.so")
SYNTH_LIB = os.path.join(PKG, "synth", "libtre_synth.so")

ENGINE_SOURCES = ["planner.cpp", "tre_api.cu", "engine.cu", "noalloc.cu"]


def engine_headers():
    """Every header in csrc/: an edit to any of them rebuilds the library."""
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".h", ".cuh")))


NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the engine needs the CUDA toolkit to build")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build_synth(force: bool = False) -> str:
    src = os.path.join(PKG, "synth", "gen.c")
    if force or _stale(SYNTH_LIB, [src]):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", src,
                               "-o", SYNTH_LIB, "-lm"])
    return SYNTH_LIB


def build_engine(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    srcs = [os.path.join(CSRC, s) for s in ENGINE_SOURCES]
    deps = srcs + [os.path.join(CSRC, h) for h in engine_headers()] + [
        os.path.join(INCLUDE, "tre.h")]
    if not (force or extra_flags or _stale(ENGINE_LIB, deps)):
        return ENGINE_LIB
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for s in srcs:
        obj = os.path.join(objdir, os.path.basename(s) + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", obj]
        if verbose and s.endswith(".cu"):
            cmd += ["-Xptxas", "-v"]
        subprocess.check_call(cmd)
        objs.append(obj)
    subprocess.check_call([nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs,
                           "-o", ENGINE_LIB, "-lcudart"])
    return ENGINE_LIB


def build_all(force: bool = False) -> None:
    build_synth(force)
    build_engine(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
    print("built", ENGINE_LIB, SYNTH_LIB)
