"""Builds libbeam_moe.so (the C ABI in include/beam_moe.h) for sm_100a with nvcc, in-tree.

Usage: ``python -m sparse_moe_transformer_fp32_b200.build [--force] [--ptxas-info]``.
Objects go to ``_build/`` at the repository root; the shared library is written next to
this file, where the Python binding loads it.  CUDA's runtime is linked statically and the
driver's tensor-map encoder is fetched at run time, so the library loads on machines without
a GPU driver (it then fails only when a call needs the device).
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libbeam_moe.so")
SOURCES = ["beam_moe_api.cu", "router.cu", "dispatch.cu", "expert_gemm.cu", "expert_gemm_2sm.cu",
           "combine.cu", "nvfp4.cu", "ep.cu"]
HEADERS = [os.path.join(CSRC, "beam_moe_internal.cuh"), os.path.join(CSRC, "beam_moe_nvfp4.cuh"),
           os.path.join(CSRC, "beam_moe_div.cuh"), os.path.join(CSRC, "beam_moe_router.cuh"),
           os.path.join(INCLUDE, "beam_moe.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    p = subprocess.run(cmd, capture_output=True, text=True)
    if p.returncode != 0:
        raise RuntimeError(f"command failed ({p.returncode}): {' '.join(cmd)}\n{p.stdout}\n{p.stderr}")
    return p.stdout + p.stderr


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    jobs = []
    objs = []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD_DIR, src.replace(".cu", ".o"))
        objs.append(o)
        if force or ptxas_info or _stale(o, [s] + HEADERS):
            extra = ["-Xptxas", "-v"] if ptxas_info else []
            jobs.append([NVCC, *ARCH, *FLAGS, *extra, "-c", s, "-o", o])
    logs = []
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            logs = list(ex.map(lambda c: _run(c, verbose), jobs))
    if force or jobs or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        _run([NVCC, *ARCH, "-shared", "-o", tmp, *objs], verbose)
        os.replace(tmp, LIB)
    if ptxas_info:
        print("\n".join(logs))
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv)
    print(LIB)
