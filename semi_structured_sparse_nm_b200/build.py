"""Builds libnmsparse.so (the C ABI of include/nmsparse.h) for sm_100a with nvcc.

The library is built in-tree next to this file.  One translation unit
(csrc/nm_api.cu) includes every kernel, so the device status word is a single
symbol.  The CUDA runtime is linked statically.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libnmsparse.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + [os.path.join(INCLUDE, "nmsparse.h")]


def nvcc_cmd(out: str, extra=()):
    return ["nvcc", "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-O2",
            "-shared", "-I", INCLUDE, "-I", CSRC, *extra,
            os.path.join(CSRC, "nm_api.cu"), "-o", out]


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    stale = (not os.path.exists(LIB)) or any(os.path.getmtime(s) > os.path.getmtime(LIB) for s in sources())
    if force or stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = nvcc_cmd(tmp, extra)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, extra=["-Xptxas", "-v"] if "-v" in sys.argv else []))
