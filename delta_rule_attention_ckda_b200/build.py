"""Build libckda.so (the CKDA C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libckda.so")
SELFTEST_LIB = os.path.join(PKG, "libckda_selftest.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


TARGETS = {LIB: "ckda_api.cu", SELFTEST_LIB: "selftest.cu"}


def _newest_input():
    files = glob.glob(os.path.join(CSRC, "**", "*.cu*"), recursive=True)
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    files.append(os.path.abspath(__file__))
    return max(os.path.getmtime(f) for f in files)


def _build_one(lib: str, src: str, force: bool, verbose: bool, extra) -> None:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_input():
        return
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           os.path.join(CSRC, src), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Build libckda.so and the test-only libckda_selftest.so; returns libckda.so's path."""
    for lib, src in TARGETS.items():
        _build_one(lib, src, force, verbose, extra)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=(["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
