"""Build libngram_embed.so in-tree for sm_100a (nvcc, no JIT cache)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libngram_embed.so")
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc_cmd(out: str, extra=()) -> list:
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    return [nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-shared", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-o", out,
            os.path.join(CSRC, "ngram_embed.cu"), *extra]


def build(force: bool = False, verbose: bool = False) -> str:
    newest = max(os.path.getmtime(f) for f in _sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    extra = ["-Xptxas", "-v"] if verbose else []
    subprocess.run(nvcc_cmd(LIB + ".tmp", extra), check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
