"""Build the in-tree CUDA library (libdp_b200.so) for sm_100a with nvcc.

Usage: python long_video_diffusion_b200/_build.py   (or __graft_entry__.build()).
The library is linked against the static CUDA runtime; the driver API entry point it
needs (tensor-map encoding) is looked up at run time, so no libcuda link is required.
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
LIB_NAME = "libdp_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

SOURCES = ["dp_api.cu", "dp_attn_tc.cu", "dp_attn_f32.cu", "dp_gemm.cu", "dp_modulate.cu", "dp_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "-shared",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, extra: list | None = None, out: str = LIB_PATH) -> str:
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    cmd = [nvcc()] + ARCH + FLAGS + (extra or []) + ["-I", INCLUDE, "-I", CSRC, "-o", out] + srcs
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed ({r.returncode})")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr)
    return out


if __name__ == "__main__":
    v = "-v" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(verbose=v, extra=extra))
