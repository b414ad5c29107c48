"""Build ``libw4b200.so`` (the whole C ABI) for sm_100a with nvcc, in-tree.

Usage: ``python -m weight_only_bit_gemm_b200.build [--verbose-ptxas]``.
Rebuilds only when a source under ``csrc/`` or ``include/`` is newer than the
library.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libw4b200.so")
# the bounds-checked build (W4_CHECKED): same functions, every kernel access
# checked against its buffer's extent (violations reported, never trapped)
LIB_CHECKED = os.path.join(PKG, "libw4b200_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def _sources():
    srcs = glob.glob(os.path.join(CSRC, "*"))
    srcs += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return srcs


def needs_build(checked: bool = False) -> bool:
    lib = LIB_CHECKED if checked else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, ptxas_verbose: bool = False, checked: bool = False) -> str:
    """Build the library (or, with checked=True, its bounds-checked twin)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(checked):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS]
    if checked:
        cmd += ["-DW4_CHECKED"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = lib + ".tmp"
    cmd += ["-o", tmp, os.path.join(CSRC, "w4_lib.cu")]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
    if "--checked" in sys.argv:
        build(force=True, checked=True)
        print(LIB_CHECKED)
