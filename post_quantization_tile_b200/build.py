"""Builds libhq.so (the CUDA codec and its C ABI) in-tree with nvcc for sm_100a, and beside it
libhq_test.so: the same library plus the test-only entry points of include/hq_test.h, whose
sources are compiled again with HQ_TEST_HOOKS (the product library carries none of them).

Usage:  python -m post_quantization_tile_b200.build      (or build() from Python)
Objects go to _build/ at the repository root; the libraries to post_quantization_tile_b200/.
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
TEST_LIB = os.path.join(PKG, "libhq_test.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         # no contraction: the encode chain is specified in binary32 without fused multiply-add
         "-fmad=false", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2", "--expt-relaxed-constexpr"]
SOURCES = ["hq_api.cu", "hq_noalloc.cu", "hq_gemm.cu", "hq_gemm_code.cu", "hq_dense.cu", "hq_inst_z.cu", "hq_inst_a2.cu", "hq_inst_d4.cu",
           "hq_inst_e8.cu"]
# sources compiled a second time with the test hooks for libhq_test.so
TEST_SOURCES = ["hq_api.cu", "hq_inst_e8.cu"]
HEADERS = ["hq_common.cuh", "hq_tc.cuh", "hq_lattice.cuh", "hq_encode.cuh", "hq_decode.cuh", "hq_instantiate.cuh", "hq_launch.h"]


def _newest_dep() -> float:
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", h) for h in ("hq.h", "hq_test.h")]
    paths.append(__file__)
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool, test: bool = False) -> str:
    out = os.path.join(OBJ, src.replace(".cu", "_test.o" if test else ".o"))
    s = os.path.join(CSRC, src)
    if os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(s), _newest_dep()):
        return out
    cmd = [NVCC, *FLAGS, *(["-DHQ_TEST_HOOKS"] if test else []), "-c", s, "-o", out]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return out


def _link(lib: str, objs: list[str], verbose: bool) -> None:
    if not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", lib, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)


def build(verbose: bool = False, jobs: int | None = None) -> str:
    os.makedirs(OBJ, exist_ok=True)
    jobs_all = [(s, False) for s in SOURCES] + [(s, True) for s in TEST_SOURCES]
    with cf.ThreadPoolExecutor(max_workers=jobs or min(len(jobs_all), os.cpu_count() or 4)) as ex:
        built = list(ex.map(lambda j: _compile(j[0], verbose, j[1]), jobs_all))
    objs = built[:len(SOURCES)]
    test_objs = dict(zip(TEST_SOURCES, built[len(SOURCES):]))
    _link(LIB, objs, verbose)
    _link(TEST_LIB, [test_objs.get(s, o) for s, o in zip(SOURCES, objs)], verbose)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
