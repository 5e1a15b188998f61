"""Build step of the CUDA library: nvcc for sm_100a, in-tree, no JIT cache."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libcsa_indexer.so")
# The debug build: kernels check their shared-memory, tensor-memory, buffer and
# output indices and report a failure through csa_last_device_error (no trap).
DEBUG_LIB = os.path.join(HERE, "libcsa_indexer_debug.so")
MAIN = os.path.join(HERE, "csrc", "csa_indexer.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    srcs = glob.glob(os.path.join(HERE, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(s) > t for s in srcs)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile ``csrc/csa_indexer.cu`` into ``libcsa_indexer.so`` next to this
    file (``debug``: ``libcsa_indexer_debug.so`` with -DCSA_DEBUG)."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DCSA_DEBUG"] if debug else []),
           "-I", os.path.join(ROOT, "include"), "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
