"""Build libqsa.so (all CUDA sources of csrc/) for sm_100a with nvcc, in-tree.

libqsa_debug.so is the same sources built with QSA_DEBUG_CHECKS: mbarrier waits
limited to 20 ms and the fault-injection site of qsa_debug_inject compiled in.
Only the failure-path tests load it (QSA_DEBUG_BUILD=1 in their child process).

Usage: python -m block_sparse_long_09_b200.build [--force] [--verbose] [--debug | --all]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libqsa.so")
LIB_DEBUG = os.path.join(HERE, "libqsa_debug.so")
DEBUG_FLAGS = ["-DQSA_DEBUG_CHECKS=1", "-DQSA_WAIT_LIMIT_NS=20000000ull"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-rdc=true",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "qsa.h")]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in deps())


def _command(lib: str, tmp: str, verbose: bool):
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc] + NVCC_FLAGS + (DEBUG_FLAGS if lib == LIB_DEBUG else []) + \
        ["-I", INCLUDE, "-I", CSRC, "-o", tmp] + sources()
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    return cmd


def build_libs(libs, force: bool = False, verbose: bool = False):
    """Build the given libraries (LIB, LIB_DEBUG) that are missing or stale, in parallel."""
    todo = [lib for lib in libs if force or needs_build(lib)]
    procs = []
    for lib in todo:
        tmp = lib + ".tmp%d" % os.getpid()
        procs.append((lib, tmp, subprocess.Popen(_command(lib, tmp, verbose))))
    failed = [lib for lib, _, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc (%s)" % ", ".join(os.path.basename(f) for f in failed))
    for lib, tmp, _ in procs:
        os.replace(tmp, lib)
    return list(libs)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    return build_libs([LIB_DEBUG if debug else LIB], force, verbose)[0]


def build_all(force: bool = False, verbose: bool = False):
    return build_libs([LIB, LIB_DEBUG], force, verbose)


if __name__ == "__main__":
    f, v = "--force" in sys.argv, "--verbose" in sys.argv
    if "--all" in sys.argv:
        print("\n".join(build_all(f, v)))
    else:
        print(build(f, v, debug="--debug" in sys.argv))
