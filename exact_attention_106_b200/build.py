"""Build the in-tree shared library ``libexattn.so`` for sm_100a with nvcc.

The library is one translation unit (``csrc/exattn.cu`` includes the kernel
headers), compiled with ``-gencode arch=compute_100a,code=sm_100a``; the CUDA
runtime is linked statically, so the library loads on a machine without a
GPU (the C-ABI exports can then be inspected, and argument checks run).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
LIB_PATH = os.path.join(PKG_DIR, "libexattn.so")
SOURCES = [os.path.join(PKG_DIR, "csrc", f) for f in ("exattn.cu", "ptx.cuh", "fwd.cuh", "bwd.cuh")]
HEADER = os.path.join(ROOT, "include", "exattn.h")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build the exattn CUDA library")


def build_command(out: str = LIB_PATH, verbose_ptxas: bool = False):
    cmd = [
        nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
        "-o", out, os.path.join(PKG_DIR, "csrc", "exattn.cu"),
    ]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def is_stale(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in SOURCES + [HEADER, __file__])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or is_stale():
        tmp = LIB_PATH + ".tmp"
        proc = subprocess.run(build_command(tmp, verbose_ptxas), capture_output=True, text=True)
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
        if verbose_ptxas:
            sys.stderr.write(proc.stderr)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
