"""Builds the two libraries in-tree with nvcc (sm_100a):

    libqsa.so        the kernels and the C ABI of include/qsa.h (production)
    libqsa_debug.so  measurement kernels and test hooks of include/qsa_debug.h,
                     compiled with QSA_DEBUG (the tests and the benchmark load
                     it next to libqsa.so; nothing in libqsa.so needs it)

    python -m top_sparse_attention_qsa_b200.build [--verbose]

Both link the CUDA runtime statically and resolve the driver at run time, so
they load on machines without a GPU (their entry points then return
QSA_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqsa.so")
DEBUG_LIB = os.path.join(PKG, "libqsa_debug.so")
DEBUG_SOURCES = ("qsa_debug_api.cu",)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def _sources(debug: bool = False):
    every = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    if debug:
        return [f for f in every if os.path.basename(f) in DEBUG_SOURCES]
    return [f for f in every if os.path.basename(f) not in DEBUG_SOURCES]


def _deps():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cu"))) + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def nvcc() -> str:
    cand = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cand, "bin", "nvcc")
    return p if os.path.exists(p) else "nvcc"


def _build_one(lib: str, debug: bool, force: bool, verbose: bool) -> str:
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    extra = ["-DQSA_DEBUG"] if debug else []
    cmd = [nvcc()] + NVCC_FLAGS + extra + ["-I", INCLUDE, "-I", CSRC, "-shared", "-o", tmp] + _sources(debug)
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds libqsa.so and (debug=True) libqsa_debug.so; returns libqsa.so's path."""
    _build_one(LIB, False, force, verbose)
    if debug:
        _build_one(DEBUG_LIB, True, force, verbose)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
