"""Build libmxq.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m mxfp4_block_rotation_b200.build [--verbose-ptxas]``.
nvcc cross-compiles without a GPU.  Each translation unit compiles to its own
object in parallel (under ``_build/``), then one link step writes the shared
library next to this file, where the Python binding loads it from.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmxq.so")
SOURCES = ["mxq_api.cu", "rotate_flat_sm100.cu", "rotate_cols_sm100.cu", "dequant_sm100.cu", "status_sm100.cu",
           "error_sm100.cu", "noalloc_sm100.cu", "search_sm100.cu", "rotate_block_sm100.cu",
           "gemm_sm100.cu"]
HEADERS = ["mxq_internal.h", "sm100_ptx.cuh", "sm100_bulk.cuh", "pipeline_sm100.cuh", "tile_order.cuh",
           os.path.join("..", "..", "include", "mxq.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _compile(src: str, verbose_ptxas: bool) -> str:
    obj = os.path.join(OBJ, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", "-o", obj, os.path.join(CSRC, src)]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not (force or verbose_ptxas or _stale()):
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        objs = list(pool.map(lambda s: _compile(s, verbose_ptxas), SOURCES))
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", LIB + ".tmp", *objs], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
