"""Build libgdr2.so in-tree with nvcc for sm_100a (no JIT, no torch extension machinery).

Usage: python -m gated_delta_rule_65_b200.build   (or call build()).
The library links the CUDA runtime statically, so it loads on a machine without a GPU driver (the
host-side argument checks can be tested there); it needs a B200 only to run kernels.
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
LIB = os.path.join(PKG, "libgdr2.so")
DEBUG_LIB = os.path.join(PKG, "libgdr2_debug.so")
SELFTEST_LIB = os.path.join(PKG, "libgdr2_selftest.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-shared",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "selftest", "*.cu")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


def build_debug(force: bool = False, verbose: bool = False) -> str:
    """libgdr2_debug.so: the library compiled with -DGDR2_DEBUG, whose kernels check their index arithmetic
    (chunk, chain, tile, TMEM and output indices) and report a failed check through gdr2_check as
    GDR2_ERR_BOUNDS instead of trapping. Used by the tests in place of a memory checker."""
    if not force and not _stale(DEBUG_LIB):
        return DEBUG_LIB
    tmp = DEBUG_LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-DGDR2_DEBUG", "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, DEBUG_LIB)
    return DEBUG_LIB


def build_selftest(force: bool = False, verbose: bool = False) -> str:
    """libgdr2_selftest.so: checks of the tcgen05 / TMA building blocks, used by the tests only."""
    if not force and not _stale(SELFTEST_LIB):
        return SELFTEST_LIB
    tmp = SELFTEST_LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp,
           os.path.join(CSRC, "selftest", "selftest.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, SELFTEST_LIB)
    return SELFTEST_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
    print(build_selftest(force="--force" in sys.argv, verbose=True))
    print(build_debug(force="--force" in sys.argv, verbose=True))
