"""Build the sm_100a shared library libindexcache.so in-tree with nvcc.

    python -m dsa_indexer_reuse_b200.build [--force] [--verbose] [--debug]

--debug builds libindexcache_debug.so instead: the same kernels compiled with
IC_DEBUG, which checks the indices that are in bounds by construction (list
appends, select outputs, compacted index rows, gathered rows) and records
IC_ERR_INTERNAL in the device status instead of accessing out of bounds.
Load it with IC_LIB_PATH=<path> before importing the package.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "indexcache.cu")
INCLUDE = os.path.join(os.path.dirname(HERE), "include", "indexcache.h")
LIB = os.path.join(HERE, "libindexcache.so")
DEBUG_LIB = os.path.join(HERE, "libindexcache_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "-diag-suppress", "177",
]


def _sources():
    files = [INCLUDE]
    for f in os.listdir(SRC_DIR):
        if f.endswith((".cu", ".cuh")):
            files.append(os.path.join(SRC_DIR, f))
    return files


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(f) for f in _sources())
        if os.path.getmtime(out) >= newest:
            return out
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = [nvcc_path(), *NVCC_FLAGS, *(["-DIC_DEBUG"] if debug else []), *(["-Xptxas", "-v"] if verbose else []),
           "-o", tmp, MAIN]
    subprocess.check_call(cmd, cwd=HERE)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
