"""Compile libusk.so for sm_100a in-tree (nvcc; no JIT cache).

    python -m sub_bit_weight_usk_b200._build
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libusk.so")
E2E = os.path.join(PKG, "usk_e2e")  # C driver: usk_gemv round trips through the C ABI alone

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh"))) + \
        sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    nvcc = os.environ.get("NVCC", "nvcc")
    if force or not up_to_date():
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-shared", "-o", tmp, *sources()]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    build_e2e(force, verbose)
    return LIB


def build_e2e(force: bool = False, verbose: bool = False) -> str:
    """The C end-to-end driver, linked against the in-tree libusk.so (rpath $ORIGIN)."""
    src = os.path.join(PKG, "driver", "usk_e2e.c")
    if not force and os.path.exists(E2E) and os.path.getmtime(E2E) >= max(os.path.getmtime(src),
                                                                           os.path.getmtime(LIB)):
        return E2E
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = E2E + ".tmp.%d" % os.getpid()
    cmd = [nvcc, "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-x", "cu", "-I", os.path.join(ROOT, "include"), "-o", tmp, src, "-L", PKG, "-lusk",
           "-Xlinker", "-rpath,$ORIGIN"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, E2E)
    return E2E


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
