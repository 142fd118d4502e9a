"""Builds the sm_100a CUDA library (csrc/attn_api.cu, one translation unit) in-tree.

    python exact_attention_ring_b200/build.py [--force] [--verbose]

produces exact_attention_ring_b200/_lib/libattn_b200.so with nvcc
``-gencode arch=compute_100a,code=sm_100a``. The CUDA runtime is linked
statically and the driver API is reached through the runtime's entry-point
query, so the library depends on nothing but the NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT_DIR = os.path.join(PKG, "_lib")
LIB_NAME = "libattn_b200.so"


def library_path() -> str:
    return os.path.join(OUT_DIR, LIB_NAME)


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(ROOT, "include", "attn.h")])


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")


def build(force: bool = False, verbose: bool = False) -> str:
    out = library_path()
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(s) for s in _sources())
        if os.path.getmtime(out) >= newest:
            return out
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), os.path.join(CSRC, "attn_api.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
