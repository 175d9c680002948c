"""Builds libdf11.so in-tree: decode.cu with nvcc for sm_100a, the host codec
and the C-ABI with g++, linked against the static CUDA runtime.

Run ``python -m entropy_decoding_b200.build`` (or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdf11.so")
INCLUDE = os.path.join(ROOT, "include")

CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

SOURCES_CU = ["decode.cu", "encode.cu", "rans_decode.cu", "gemm.cu"]
SOURCES_CPP = ["codec.cpp", "capi.cpp", "rans.cpp"]
HEADERS = ["df11_internal.h", "codec.h", "launch.h", "encode.h", "rans.h", "walk.cuh", "gemm.h"]


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
          extra_nvcc: list[str] | None = None) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "df11.h")]
    objs = []
    for src in SOURCES_CU:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        if force or ptxas_verbose or _newer(o, [s] + hdrs):
            cmd = [NVCC, *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
                   "-I", INCLUDE, "-c", s, "-o", o]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            cmd += extra_nvcc or []
            _run(cmd, verbose)
        objs.append(o)
    for src in SOURCES_CPP:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        if force or _newer(o, [s] + hdrs):
            _run(["g++", "-O3", "-std=c++17", "-fPIC", "-Wall", "-Wextra", "-pthread",
                  "-I", os.path.join(CUDA_HOME, "include"), "-I", INCLUDE, "-c", s, "-o", o], verbose)
        objs.append(o)
    if force or _newer(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        _run([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lpthread", "-ldl", "-lrt"],
             verbose)
        os.replace(tmp, LIB)
    return LIB


def clean():
    shutil.rmtree(BUILD, ignore_errors=True)
    if os.path.exists(LIB):
        os.remove(LIB)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_verbose="-v" in sys.argv)
