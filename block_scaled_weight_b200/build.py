"""Build ``libmxq.so`` in-tree with nvcc for sm_100a (B200).

The library is a plain C-ABI shared object (see ``include/mxq.h``); the CUDA runtime is
linked statically so the object carries no dependency on any particular libcudart. Every
kernel is the library's own; no CUDA math library is linked.
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmxq.so")
SOURCES = ["mxq_api.cu", "mxq_hpass.cu", "mxq_gram.cu", "mxq_quant.cu", "mxq_quant_grid.cu",
           "mxq_error.cu", "mxq_outerr.cu", "mxq_gptq.cu", "mxq_gptq_full.cu", "mxq_gram_full.cu",
           "mxq_nvfp4_mm.cu",
           "mxq_noalloc.cu"]
HEADERS = ["mxq_common.cuh", "mxq_internal.h", "mxq_block.cuh", "mxq_grids.h", "mxq_gridk.cuh",
           "mxq_chol64.cuh", "mxq_tc.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "mxq.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every translation unit and link ``libmxq.so`` next to this file."""
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(ROOT, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = [os.path.join(objdir, src.replace(".cu", ".o")) for src in SOURCES]

    def compile_one(src, obj):
        cmd = [nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)

    # the translation units are independent: compile them side by side
    workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as pool:
        for f in [pool.submit(compile_one, s, o) for s, o in zip(SOURCES, objs)]:
            f.result()
    tmp = LIB + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-cudart", "static"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
