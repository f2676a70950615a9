"""Build libjetlong.so in-tree with nvcc for sm_100a.

    python -m zero_shot_rope_bifocal_b200.build        # incremental
    python -m zero_shot_rope_bifocal_b200.build --force

Each CUDA source compiles to an object under ``_build/`` at the repository
root; the objects link (static CUDA runtime) into
``zero_shot_rope_bifocal_b200/libjetlong.so``.  The library needs only the
NVIDIA driver at run time, and loads without one (CUDA initialises lazily on
the first device call).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libjetlong.so")
SOURCES = ["jetlong_api.cu", "rope_kernels.cu", "decode_kernels.cu", "prefill_sm100.cu",
           "three_pass.cu"]
HEADERS = ["jl_common.cuh", "sm100_ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def _mtime(p: str) -> float:
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    header_time = max(_mtime(os.path.join(CSRC, h)) for h in HEADERS)
    header_time = max(header_time, _mtime(os.path.join(ROOT, "include", "jetlong.h")))
    objs = []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        op = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(op)
        if force or _mtime(op) < max(_mtime(sp), header_time):
            cmd = [nvcc(), *ARCH, *CFLAGS, "-c", sp, "-o", op]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _mtime(LIB) < max(_mtime(o) for o in objs):
        # Export only the C ABI: every other symbol keeps hidden visibility.
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-Xcompiler", "-fPIC", *objs, "-o", LIB]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))
    return 0


if __name__ == "__main__":
    sys.exit(main())
