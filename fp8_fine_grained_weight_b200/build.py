"""Build ``libfp8q.so`` (the C ABI of include/fp8q.h) in-tree with nvcc for sm_100a.

``python -m fp8_fine_grained_weight_b200.build`` or :func:`build`.  Cross-compiles on a
machine without a GPU.  No fast-math: the quantizers' division and rounding are part
of their bit-exact contract.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8q.so")
SOURCES = [os.path.join(CSRC, "fp8q.cu")]


def deps() -> list:
    """Every file the library is built from: the sources, every header under csrc/ and the
    public header.  A change to any of them makes the next build() recompile."""
    hdrs = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))
    return SOURCES + hdrs + [os.path.join(ROOT, "include", "fp8q.h")]


ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def command(out: str = LIB, extra=()) -> list:
    return [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-Xptxas", "-v", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
            *extra, "-o", out, *SOURCES]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in deps()):
            return LIB
    tmp = LIB + ".tmp"
    res = subprocess.run(command(tmp), capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libfp8q.so")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
