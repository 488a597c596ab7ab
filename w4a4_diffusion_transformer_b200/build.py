"""Build the in-tree shared library ``libsvdq.so`` for sm_100a.

CUDA sources are compiled with ``nvcc -gencode arch=compute_100a,code=sm_100a``
(no GPU is needed to build), the host preparation code with ``g++ -fopenmp``,
and everything is linked into ``w4a4_diffusion_transformer_b200/libsvdq.so``
next to this file.  Objects go to ``_build/`` at the repository root; a source
is recompiled only when it or a header changed.

    python -m w4a4_diffusion_transformer_b200.build [--force]
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsvdq.so")

CUDA_SOURCES = ["api.cu", "k1_quant.cu", "k2_gemm.cu", "k2_pair.cu", "k2_int4.cu", "k2_int4_pair.cu", "upproj.cu", "static_ws.cu", "w4a16.cu", "selftest.cu", "chain.cu", "k2_int8.cu"]
CXX_SOURCES = ["prepare.cpp"]
HEADERS = [os.path.join(CSRC, h) for h in ("sm100.cuh", "kernels.h", "svdq_internal.h", "nvfp4_quant.cuh")] + [
    os.path.join(INCLUDE, "svdq.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
              "--expt-relaxed-constexpr", "-I", INCLUDE]
CXX_FLAGS = ["-std=c++17", "-O3", "-fPIC", "-fopenmp", "-ffp-contract=off", "-mavx2", "-mfma",
             "-I", INCLUDE]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else (shutil.which("nvcc") or "nvcc")


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + HEADERS)


def _run(cmd, log):
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    log.append(r.stdout)
    if r.returncode != 0:
        raise RuntimeError(f"build step failed: {' '.join(cmd)}\n{r.stdout}")
    return r.stdout


def _compile(cmd, obj, log):
    """One compile into a temporary object, renamed into place on success, so
    an interrupted build never leaves a truncated object that looks fresh."""
    tmp = obj + ".tmp"
    _run(cmd + ["-o", tmp], log)
    os.replace(tmp, obj)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source for sm_100a and link libsvdq.so; returns its path.
    Stale sources compile in parallel (one process each)."""
    from concurrent.futures import ThreadPoolExecutor

    os.makedirs(BUILD, exist_ok=True)
    log: list = []
    objs, jobs = [], []
    changed = force or not os.path.exists(LIB)
    for src in CUDA_SOURCES + CXX_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, s):
            cxx = src in CXX_SOURCES
            cmd = (["g++"] + CXX_FLAGS if cxx else [_nvcc()] + ARCH + NVCC_FLAGS) + ["-c", s]
            jobs.append((cmd, o))
    if jobs:
        logs = [[] for _ in jobs]
        with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as pool:
            futures = [pool.submit(_compile, cmd, o, lg) for (cmd, o), lg in zip(jobs, logs)]
            errors = [f.exception() for f in futures]
        for lg in logs:
            log.extend(lg)
        failed = [e for e in errors if e is not None]
        if failed:
            raise failed[0]
        changed = True
    if changed or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        tmp = LIB + ".tmp"
        _run([_nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-Xcompiler", "-fopenmp", "-lgomp"], log)
        os.replace(tmp, LIB)
    if verbose:
        print("".join(log))
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
