"""Build ``libbsa.so`` in-tree: the sm_100a kernel plus the host C ABI.

Run as ``python -m block_sparse_long_bsa_b200.build`` (or through
``__graft_entry__.build()``).  nvcc cross-compiles sm_100a without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libbsa.so")

CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]

CU_SOURCES = ["bsa_fwd_sm100a.cu", "bsa_noalloc.cu", "bsa_decode.cu", "bsa_bwd_sm100a.cu", "bsa_bsbr_sm100a.cu"]
CPP_SOURCES = ["bsa_api.cpp", "bsa_layout.cpp", "bsa_tmap.cpp"]
HEADERS = [os.path.join(INCLUDE, "bsa.h"), os.path.join(CSRC, "bsa_internal.h"), os.path.join(CSRC, "bsa_device.cuh"),
           os.path.join(CSRC, "bsa_tmap.h")]


def _newer(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if verbose and res.stdout.strip():
        print(res.stdout, flush=True)
    if res.returncode != 0:
        raise RuntimeError(f"build step failed ({res.returncode}): {' '.join(cmd)}\n{res.stdout}")
    return res.stdout


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    common = ["-O3", "-std=c++17", f"-I{INCLUDE}", f"-I{CSRC}"]
    for src in CU_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        if force or ptxas_info or _newer(o, [s] + HEADERS):
            cmd = [NVCC] + ARCH + common + ["-lineinfo", "-Xcompiler", "-fPIC", "-c", s, "-o", o]
            if ptxas_info:
                cmd.insert(1, "-Xptxas=-v")
            _run(cmd, verbose or ptxas_info)
        objs.append(o)
    for src in CPP_SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        if force or _newer(o, [s] + HEADERS):
            cxx = shutil.which("g++") or "g++"
            _run([cxx, "-O2", "-std=c++17", "-fPIC", "-Wall", f"-I{INCLUDE}", f"-I{CSRC}",
                  f"-I{os.path.join(CUDA_HOME, 'include')}", "-c", s, "-o", o], verbose)
        objs.append(o)
    if force or _newer(LIB, objs):
        _run([NVCC] + ARCH + ["-shared", "-cudart", "static", "-o", LIB] + objs +
             ["-Xlinker", "--no-undefined"], verbose)
    return LIB


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv, ptxas_info="--ptxas" in sys.argv)
