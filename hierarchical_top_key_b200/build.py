"""Build libhisa.so in-tree with nvcc for sm_100a.

    python -m hierarchical_top_key_b200.build [--force] [--verbose-ptxas]

The library is a single translation unit (csrc/libhisa.cu includes every
kernel header) linked against the static CUDA runtime, so the .so carries no
dependency on a particular libcudart and ships with the source tree.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libhisa.so")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(ROOT, "include", "hisa.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [
        nvcc_path(), "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "--expt-relaxed-constexpr", "--extended-lambda",
        "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
        "-shared", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"),
        os.path.join(CSRC, "libhisa.cu"),
        "-o", LIB + ".tmp",
    ]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    if debug:
        cmd.insert(1, "-DHISA_DEBUG=1")
    print("[hisa build]", " ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas))


if __name__ == "__main__":
    main()
