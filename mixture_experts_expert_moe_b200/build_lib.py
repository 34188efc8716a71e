"""Build libmoe_b200.so (the C-ABI library) in-tree for sm_100a with nvcc.

Usage: python -m mixture_experts_expert_moe_b200.build_lib [-v] [--debug]

``--debug`` builds libmoe_b200_debug.so instead: the same kernels compiled
with MOE_DEBUG, whose index checks skip an out-of-range access and report
MOE_DEV_BOUNDS in the device status word.  The binding loads it when the
environment variable MOE_B200_LIB names its path.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")
DEBUG_BUILD = os.path.join(PKG, "_build_debug")
DEBUG_LIB = os.path.join(PKG, "libmoe_b200_debug.so")
SOURCES = ["api.cu", "align_sort.cu", "bwd.cu", "elementwise.cu", "grouped_gemm.cu", "mx.cu", "noalloc.cu"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "-I" + os.path.join(ROOT, "include"),
]


def _compile(src: str, verbose_ptxas: bool, debug: bool) -> str:
    obj = os.path.join(DEBUG_BUILD if debug else BUILD, src.replace(".cu", ".o"))
    cmd = [NVCC, *FLAGS, *(["-DMOE_DEBUG"] if debug else []), "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def build(verbose_ptxas: bool = False, debug: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    os.makedirs(DEBUG_BUILD if debug else BUILD, exist_ok=True)
    if os.path.exists(out):
        os.remove(out)   # never leave a stale library behind a failed build
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, debug), SOURCES))
    cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
           *objs, "-o", out, "-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return out


if __name__ == "__main__":
    print(build(verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))
