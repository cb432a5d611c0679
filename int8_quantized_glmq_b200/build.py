"""Build the glmq shared library (CUDA C++ for sm_100a) in-tree.

    python -m int8_quantized_glmq_b200.build        # builds int8_quantized_glmq_b200/libglmq.so

The library is one translation unit (csrc/glmq.cu) compiled by nvcc for
sm_100a only, with the CUDA runtime linked statically. No fast-math: the
quantizer's exact rounding depends on IEEE division and rounding behaviour.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "glmq.cu")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libglmq.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the glmq library needs the CUDA toolkit to build")


def sources():
    csrc = os.path.join(PKG, "csrc")
    out = [os.path.join(csrc, f) for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh"))]
    out.append(os.path.join(INCLUDE, "glmq.h"))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-o", LIB + ".tmp", SRC]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
