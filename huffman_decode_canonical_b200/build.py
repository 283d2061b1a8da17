"""Build libentro.so in-tree with nvcc for sm_100a (B200).

    python huffman_decode_canonical_b200/build.py [--verbose-ptxas]

(Run it as a script: importing the package itself loads libentro.so.)

The shared library lands next to this file, so it travels with the source
tree.  Host code is compiled without floating-point contraction so that the
encoder's quantization is reproducible bit for bit.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libentro.so")
SOURCES = [os.path.join(CSRC, "decode.cu"), os.path.join(CSRC, "encoder.cpp")]
HEADERS = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))) + [
    os.path.join(ROOT, "include", "entro.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC,-pthread,-ffp-contract=off,-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", tmp] + SOURCES + ["-lpthread"]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
