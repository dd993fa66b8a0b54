"""Build the BitLinear CUDA library in-tree for sm_100a.

    python -m int8_row_absmax_b200.build        # -> int8_row_absmax_b200/libbitlinear.so

One nvcc invocation over one translation unit.  No fast-math: the quantizers
need IEEE division and round-half-even, and -fmad=false keeps the dequant
epilogue from being contracted into an FMA.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "bitlinear_lib.cu")
OUT = os.path.join(PKG, "libbitlinear.so")
ARCH = "-gencode=arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    d = os.path.join(PKG, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + \
        [os.path.join(ROOT, "include", "bitlinear.h")]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return OUT
    cmd = [nvcc_path(), ARCH, "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
           "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-warn-spills",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc"),
           *extra, "-o", OUT + ".tmp", SRC]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force or bool(extra), verbose=True, extra=extra))
