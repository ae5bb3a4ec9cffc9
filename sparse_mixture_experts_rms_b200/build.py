"""Build the sm_100a shared library ``libmoe_b200.so`` in-tree with nvcc.

    python -m sparse_mixture_experts_rms_b200.build

The CUDA runtime is linked statically and the driver entry point for TMA
descriptor encoding is fetched at run time, so the library loads (and its
host-side argument checks run) on machines without a GPU driver.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)

SOURCES = ["moe_api.cu", "route.cu", "dispatch.cu", "grouped_gemm.cu", "combine.cu", "backward.cu", "quantize.cu", "grouped_gemm_mx.cu", "api_train.cu", "api_mx.cu",
           "api_host.cu"]
HEADERS = ["moe_internal.h", "api_detail.h", "ptx.cuh", "mx.cuh", "pair_pipe.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libmoe_b200.so")
    return cand


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "moe.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile every CUDA source for sm_100a into one shared library."""
    if not force and up_to_date():
        return LIB_PATH
    nvcc = _nvcc()
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, *(extra_flags or []), "-shared", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr, file=sys.stderr)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    force = "--force" in sys.argv
    p = build(force=force, verbose=True,
              extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(p)
