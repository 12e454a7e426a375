"""Build libw8a16.so in-tree with nvcc for sm_100a (B200).

    python -m int8_weight_only_b200.build [--verbose]

Compiles csrc/w8a16.cu (which includes every kernel) into
int8_weight_only_b200/libw8a16.so.  No GPU is needed to build.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "w8a16.cu")
HEADER = os.path.join(ROOT, "include", "w8a16.h")
LIB = os.path.join(HERE, "libw8a16.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    # IEEE division and denormals are required for bit-exact quantization
    "-prec-div=true", "-ftz=false", "-prec-sqrt=true", "-fmad=true",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    out = [HEADER]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-o", tmp, MAIN]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd, cwd=ROOT)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
