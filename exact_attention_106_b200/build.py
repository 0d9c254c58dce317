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
# ptxas's per-kernel resource report of the last build (registers, spills)
RESOURCES_PATH = os.path.join(PKG_DIR, "libexattn.resources.txt")
SOURCES = [os.path.join(PKG_DIR, "csrc", f) for f in ("exattn.cu", "ptx.cuh", "fwd.cuh", "bwd.cuh")]
HEADER = os.path.join(ROOT, "include", "exattn.h")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: cannot build the exattn CUDA library")


def build_command(out: str = LIB_PATH, cudart: str = "static"):
    """nvcc command line for the library.  ``cudart="shared"`` links the CUDA
    runtime dynamically instead (the tests use such a build to share one
    runtime with a caller that resets the device)."""
    return [
        nvcc_path(), "-Xptxas", "-v", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
        "-std=c++17", "-Xcompiler", "-fPIC", "-shared", f"-cudart={cudart}", "-I", os.path.join(ROOT, "include"),
        "-o", out, os.path.join(PKG_DIR, "csrc", "exattn.cu"),
    ]


def is_stale(out: str = LIB_PATH) -> bool:
    if not os.path.exists(out) or not os.path.exists(RESOURCES_PATH):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in SOURCES + [HEADER, __file__])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or is_stale():
        tmp = LIB_PATH + ".tmp"
        proc = subprocess.run(build_command(tmp), capture_output=True, text=True)
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
        if verbose_ptxas:
            sys.stderr.write(proc.stderr)
        report = [ln for ln in proc.stderr.splitlines() if "ptxas info" in ln or "bytes stack frame" in ln]
        with open(RESOURCES_PATH + ".tmp", "w") as f:
            f.write("\n".join(report) + "\n")
        os.replace(tmp, LIB_PATH)
        os.replace(RESOURCES_PATH + ".tmp", RESOURCES_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
