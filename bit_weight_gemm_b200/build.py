"""Builds libbonsai.so in-tree with nvcc for sm_100a.

Run as ``python -m bit_weight_gemm_b200.build`` or call ``build()``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libbonsai.so")
MAIN = os.path.join(HERE, "csrc", "bonsai.cu")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*"))) + [os.path.join(ROOT, "include", "bonsai.h")]


def command(out: str = LIB, extra: list[str] | None = None) -> list[str]:
    return [
        NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
        "-I", os.path.join(ROOT, "include"),
        *(extra or []),
        "-o", out, MAIN,
    ]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = not os.path.exists(LIB) or any(os.path.getmtime(s) > os.path.getmtime(LIB) for s in sources())
    if force or stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = command(tmp, ["-Xptxas", "-v"] if verbose else None)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
