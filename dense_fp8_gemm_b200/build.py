"""Build the Spense CUDA library (libspense.so) in-tree for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libspense.so")
# The same library with the failure-path test hook compiled in (SPENSE_TEST_HOOKS:
# SPENSE_TEST_STALL=1 makes the GEMM's loaders wait on a word nothing sets).
# Only the failure tests load it; the product library has no such hook.
TEST_LIB_PATH = os.path.join(LIB_DIR, "libspense_testhooks.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra=(), path: str = LIB_PATH) -> str:
    if not force and up_to_date(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC, *extra, *sources(),
           "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, path)
    return path


def build_test_hooks(force: bool = False, verbose: bool = False) -> str:
    """libspense_testhooks.so: the library with SPENSE_TEST_HOOKS defined."""
    return build(force=force, verbose=verbose, extra=("-DSPENSE_TEST_HOOKS",), path=TEST_LIB_PATH)


if __name__ == "__main__":
    print(build(force=True, verbose=True, extra=sys.argv[1:]))
