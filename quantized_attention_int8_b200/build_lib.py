"""Builds the CUDA library in-tree with nvcc for sm_100a: libsage_b200.so and its checked
twin libsage_b200_checked.so (-DSAGE_CHECKED: every kernel store tests its extent first).

Usage: python quantized_attention_int8_b200/build_lib.py [--force] [--ptxas-info] [--no-checked]

Run it as a script (not as a module of the package): importing the package
loads the library, which may not exist yet or may be stale.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsage_b200.so")
LIB_CHECKED = os.path.join(PKG, "libsage_b200_checked.so")
SOURCES = ["api.cu", "attn.cu", "quant.cu"]
HEADERS = ["sm100.cuh", "sage_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsage_b200.so")
    return cand


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sage.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def _build_one(lib: str, defines: list[str], force: bool, ptxas_info: bool, verbose: bool) -> str:
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-shared",
           "--threads", "4", *defines, f"-I{INCLUDE}", f"-I{CSRC}", "-o", tmp,
           *[os.path.join(CSRC, f) for f in SOURCES]]
    if ptxas_info:
        cmd[1:1] = ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if ptxas_info or verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False, checked: bool = True) -> str:
    """Builds the library (and, unless checked=False, its checked twin); returns the library's path."""
    _build_one(LIB, [], force, ptxas_info, verbose)
    if checked:
        _build_one(LIB_CHECKED, ["-DSAGE_CHECKED"], force, ptxas_info, verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_info="--ptxas-info" in sys.argv, verbose=True,
          checked="--no-checked" not in sys.argv)
