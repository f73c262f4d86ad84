"""Builds the CUDA library ``librf2.so`` in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librf2.so")
SOURCES = ["rf2_lib.cu"]
DEPS = ["rf2_lib.cu", "attn.cuh", "mask.cuh", "topn.cuh", "permute.cuh", "geometry.cuh", "ptx.cuh"]


def nvcc_cmd(out: str, extra=()) -> list:
    return [
        "nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-Xptxas", "-v", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC, *extra,
        "-o", out, *[os.path.join(CSRC, s) for s in SOURCES],
    ]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "rf2.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        tmp = LIB + ".tmp"
        r = subprocess.run(nvcc_cmd(tmp), capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed building librf2.so")
        if verbose:
            sys.stderr.write(r.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose=True)
    print(LIB)
