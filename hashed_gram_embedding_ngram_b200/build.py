"""Build libngram.so in-tree with nvcc for sm_100a (B200).

    python hashed_gram_embedding_ngram_b200/build.py [--force]

It is a standalone script (it does not import the package, whose import needs the
library it builds).

The shared library lands next to this file so that it travels with the source tree;
ptxas resource usage (registers, spills, shared memory) is written to
``_build/ptxas.txt`` in this directory.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libngram.so")
BUILD_DIR = os.path.join(HERE, "_build")

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden,-fopenmp",
    "-Xptxas", "-v",
    "-shared",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) +
            sorted(glob.glob(os.path.join(INCLUDE, "*.h"))))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-o", tmp, *_sources(), "-lgomp"]
    p = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(BUILD_DIR, "ptxas.txt"), "w") as f:
        f.write(" ".join(cmd) + "\n" + p.stdout + p.stderr)
    if p.returncode != 0:
        sys.stderr.write(p.stdout + p.stderr)
        raise RuntimeError("nvcc failed building libngram.so (exit %d)" % p.returncode)
    if verbose:
        sys.stdout.write(p.stdout + p.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
