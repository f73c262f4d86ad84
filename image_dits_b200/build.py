"""Builds the CUDA library ``librf2.so`` in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librf2.so")
CHECKED_LIB = os.path.join(HERE, "librf2_checked.so")
SOURCES = ["rf2_lib.cu"]
DEPS = ["rf2_lib.cu", "attn.cuh", "mask.cuh", "topn.cuh", "permute.cuh", "geometry.cuh", "ptx.cuh"]


def nvcc_cmd(out: str, extra=()) -> list:
    return [
        "nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-Xptxas", "-v", "-shared", "-Xcompiler", "-fPIC", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC, *extra,
        "-o", out, *[os.path.join(CSRC, s) for s in SOURCES],
    ]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(ROOT, "include", "rf2.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def _build_one(lib: str, extra, force: bool, verbose: bool):
    if force or _stale(lib):
        tmp = lib + ".tmp"
        r = subprocess.run(nvcc_cmd(tmp, extra), capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
        if verbose:
            sys.stderr.write(r.stderr)
        os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds librf2.so and its range-checked twin librf2_checked.so
    (RF2_CHECKED=1: the same code plus index checks reported through the
    device status word); returns the path of librf2.so."""
    _build_one(LIB, (), force, verbose)
    _build_one(CHECKED_LIB, ("-DRF2_CHECKED=1",), force, verbose)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose=True)
    print(LIB, CHECKED_LIB)
