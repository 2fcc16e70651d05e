"""Build the sm_100a CUDA library libllmint8.so in-tree with nvcc.

The library exposes only the C ABI of include/llmint8.h. It is compiled for
sm_100a alone (tcgen05 / TMA code has no other target) with IEEE division
(no fast math), which the bit-exact quantisation relies on.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libllmint8.so")
SOURCES = [os.path.join(CSRC, "llmint8_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith(".cuh")] + [os.path.join(INCLUDE, "llmint8.h")]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def nvcc_flags(verbose_ptxas: bool = False):
    flags = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
             "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
             "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    return flags


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in DEPS)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path()] + nvcc_flags(verbose_ptxas) + ["-shared", "-o", tmp] + SOURCES
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
