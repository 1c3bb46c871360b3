"""Build the sm_100a shared library ``libbasiskv.so`` in-tree with nvcc.

    python -m compressed_kv_cache_routing_b200.build [--force]
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libbasiskv.so")
HEADER = os.path.join(ROOT, "include", "basiskv.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-shared",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


# The wait-expiry test build: the same sources with BASISKV_WAIT_TEST, which
# shortens every bounded wait to 1 ms and has one warp skip one copy, so a
# test can watch a wait run out and the kernels return with a status (no
# fault, no hang).  It holds only the Llama-3-8B decode shapes.
WAIT_TEST_LIB = os.path.join(HERE, "libbasiskv_waittest.so")


def _stale_lib(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER, __file__]
    return any(os.path.getmtime(f) > t for f in deps)


def _stale() -> bool:
    return _stale_lib(LIB)


def _compile(lib: str, extra: list[str], verbose: bool) -> str:
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    return _compile(LIB, [], verbose)


# The debug build: the same sources with BASISKV_DEBUG, which checks the
# indices the kernels keep in range by construction (ring stage, unit, KV
# head, pool row, score and selection entries) and records
# BASISKV_STATUS_DEBUG_BOUNDS instead of making a bad access.
DEBUG_LIB = os.path.join(HERE, "libbasiskv_debug.so")


def build_debug(force: bool = False) -> str:
    if not force and not _stale_lib(DEBUG_LIB):
        return DEBUG_LIB
    return _compile(DEBUG_LIB, ["-DBASISKV_DEBUG"], False)


def build_wait_test(force: bool = False) -> str:
    if not force and not _stale_lib(WAIT_TEST_LIB):
        return WAIT_TEST_LIB
    return _compile(WAIT_TEST_LIB, ["-DBASISKV_WAIT_TEST"], False)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
