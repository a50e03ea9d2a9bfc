"""Build libgqa.so in-tree with nvcc for sm_100a (B200).

    python -m kv_cache_02_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libgqa.so")
MAIN = os.path.join(HERE, "csrc", "gqa_lib.cu")
UNITS = [MAIN, os.path.join(HERE, "csrc", "decode_noalloc.cu")]

# A second build of the same sources for one GPU test of the failure path:
# bounded waits give up after 20 ms instead of 1 s, and the first CTA of a
# narrow-group decode never loads its first item's second tile, so its
# consumers' wait for that tile runs out (GQA_DEVERR_TIMEOUT). Nothing but
# tests/test_gpu_wait_timeout.py loads it.
WAIT_TEST_LIB = os.path.join(HERE, "libgqa_waittest.so")
WAIT_TEST_FLAGS = ["-DGQA_WAIT_TEST", "-DGQA_WAIT_LIMIT_NS=20000000ull"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources() -> list:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*")) + [os.path.join(ROOT, "include", "gqa.h")])


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(lib: str, units, flags, force: bool, verbose: bool) -> str:
    stale = not os.path.exists(lib) or any(os.path.getmtime(s) > os.path.getmtime(lib) for s in sources())
    if not (force or stale):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-o", tmp, *units]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Build libgqa.so and the wait-test library; returns the path of libgqa.so."""
    _build_one(WAIT_TEST_LIB, [MAIN], [*WAIT_TEST_FLAGS, *extra], force, verbose)
    return _build_one(LIB, UNITS, list(extra), force, verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
    print(LIB)
