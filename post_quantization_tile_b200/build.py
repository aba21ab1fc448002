"""Builds libhq.so (the CUDA codec and its C ABI) in-tree with nvcc for sm_100a.

Usage:  python -m post_quantization_tile_b200.build      (or build() from Python)
Objects go to _build/ at the repository root; the library to post_quantization_tile_b200/libhq.so.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libhq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         # no contraction: the encode chain is specified in binary32 without fused multiply-add
         "-fmad=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2", "--expt-relaxed-constexpr"]
SOURCES = ["hq_api.cu", "hq_noalloc.cu", "hq_gemm.cu", "hq_dense.cu", "hq_inst_z.cu", "hq_inst_a2.cu", "hq_inst_d4.cu",
           "hq_inst_e8.cu"]
HEADERS = ["hq_common.cuh", "hq_lattice.cuh", "hq_encode.cuh", "hq_decode.cuh", "hq_instantiate.cuh", "hq_launch.h"]


def _newest_dep() -> float:
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "hq.h"), __file__]
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool) -> str:
    out = os.path.join(OBJ, src.replace(".cu", ".o"))
    s = os.path.join(CSRC, src)
    if os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(s), _newest_dep()):
        return out
    cmd = [NVCC, *FLAGS, "-c", s, "-o", out]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return out


def build(verbose: bool = False, jobs: int | None = None) -> str:
    os.makedirs(OBJ, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=jobs or min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), SOURCES))
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", LIB, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
