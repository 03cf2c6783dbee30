"""Builds the C-ABI shared library libdm05_suffix_attn.so in-tree (sm_100a)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdm05_suffix_attn.so")
SOURCES = [os.path.join(HERE, "csrc", "dm05_suffix_attn.cu")]


def deps() -> list:
    """Every file the library is compiled from: the sources, each header the
    sources include from csrc/, and the public header."""
    csrc = os.path.join(HERE, "csrc")
    inc = os.path.join(ROOT, "include")
    out = list(SOURCES)
    for d, exts in ((csrc, (".cuh", ".h")), (inc, (".h",))):
        out += [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith(exts)]
    return out


NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile when the library is missing or older than a source file."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in deps()):
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True)
