"""Builds libdf11.so in-tree: the kernels with nvcc for sm_100a, the host
codec and the C-ABI with g++, linked against the static CUDA runtime; and
libdf11_check.so, the same library with the kernels compiled with
-DDF11_CHECK=1 (every table, stage, exponent-buffer and section access of the
decode checked; a violation sets DF11_DEV_ERR_BOUNDS and is skipped).

Run ``python -m entropy_decoding_b200.build [--check]`` (or
``__graft_entry__.build()``, which builds both).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdf11.so")
BUILD_CHECK = os.path.join(HERE, "_build_check")
LIB_CHECK = os.path.join(HERE, "libdf11_check.so")
INCLUDE = os.path.join(ROOT, "include")

CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

SOURCES_CU = ["decode.cu", "encode.cu", "rans_decode.cu", "gemm.cu"]
SOURCES_CPP = ["codec.cpp", "capi.cpp", "rans.cpp"]
HEADERS = ["df11_internal.h", "codec.h", "launch.h", "encode.h", "rans.h", "walk.cuh", "gemm.h", "merge.cuh", "check.cuh"]


def _newer(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd: list[str], verbose: bool):
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          extra_nvcc: list[str] | None = None, check: bool = False) -> str:
    """Builds libdf11.so (check=False) or libdf11_check.so (check=True) and
    returns its path.  The host objects are shared by both."""
    lib = LIB_CHECK if check else LIB
    cu_dir = BUILD_CHECK if check else BUILD
    os.makedirs(BUILD, exist_ok=True)
    os.makedirs(cu_dir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "df11.h")]
    jobs, objs = [], []
    for src in SOURCES_CU:
        s = os.path.join(CSRC, src)
        o = os.path.join(cu_dir, src + ".o")
        if force or ptxas_verbose or _newer(o, [s] + hdrs):
            cmd = [NVCC, *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                   "-I", INCLUDE, "-c", s, "-o", o]
            if check:
                cmd += ["-DDF11_CHECK=1"]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            cmd += extra_nvcc or []
            jobs.append(cmd)
        objs.append(o)
    for src in SOURCES_CPP:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        if force or _newer(o, [s] + hdrs):
            jobs.append(["g++", "-O3", "-std=c++17", "-fPIC", "-Wall", "-Wextra", "-pthread",
                         "-I", os.path.join(CUDA_HOME, "include"), "-I", INCLUDE, "-c", s, "-o", o])
        objs.append(o)
    if jobs:
        with ThreadPoolExecutor(max_workers=min(len(jobs), max(1, os.cpu_count() or 1))) as ex:
            for f in [ex.submit(_run, cmd, verbose) for cmd in jobs]:
                f.result()
    if force or _newer(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        _run([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lpthread", "-ldl", "-lrt"],
             verbose)
        os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> tuple[str, str]:
    """Both libraries: libdf11.so and libdf11_check.so."""
    return build(force=force, verbose=verbose), build(force=force, verbose=verbose, check=True)


def clean():
    for d in (BUILD, BUILD_CHECK):
        shutil.rmtree(d, ignore_errors=True)
    for f in (LIB, LIB_CHECK):
        if os.path.exists(f):
            os.remove(f)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_verbose="-v" in sys.argv, check="--check" in sys.argv)
