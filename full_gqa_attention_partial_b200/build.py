"""Builds the CUDA library in-tree: full_gqa_attention_partial_b200/_lib/libhyb_attn.so.

nvcc cross-compiles for sm_100a without a GPU.  The whole library is one
translation unit (csrc/hyb_attn_lib.cu).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libhyb_attn.so")
# the same library with -DHYB_DEBUG_BOUNDS: device-side index checks that report
# through the error word (HYB_DEV_ERR_BOUNDS) and skip the access
DEBUG_LIB = os.path.join(LIB_DIR, "libhyb_attn_debug.so")


def sources() -> list:
    """Every file under csrc/ (the unity build includes them all)."""
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".h")))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(ROOT, "include", "hyb_attn.h")]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _compile(lib: str, defines: list, verbose: bool) -> None:
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = lib + ".tmp"
    cmd = [
        nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
        "-Xptxas", "-v" if verbose else "-O3", *defines,
        "-o", tmp, os.path.join(CSRC, "hyb_attn_lib.cu"),
    ]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, lib)


def build(verbose: bool = False, force: bool = False, debug: bool = True) -> str:
    """Builds the library (and, with debug, its -DHYB_DEBUG_BOUNDS twin); returns the normal one's path."""
    if force or needs_build(LIB):
        _compile(LIB, [], verbose)
    if debug and (force or needs_build(DEBUG_LIB)):
        _compile(DEBUG_LIB, ["-DHYB_DEBUG_BOUNDS"], verbose)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
