"""Builds libmoe_b200.so in-tree with nvcc for sm_100a.

    python -m mixture_experts_expert_route_b200.build [--verbose-ptxas] [--debug-checks]

--debug-checks builds libmoe_b200_debug.so instead: the same library compiled
with MOE_DEBUG_CHECKS, whose kernels validate the permutation they are handed
and report a bad entry in the status word (MOE_ERR_DEVICE).  The binding
loads it when the environment sets MOE_B200_DEBUG_CHECKS=1.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["route_permute.cu", "elementwise.cu", "grouped_gemm.cu", "moe_api.cu", "noalloc.cu",
           "split.cu"]
# host code of the CPU/GPU split (g++: the AVX512_BF16 kernel selects its
# instruction set per function and checks the CPU at run time)
HOST_SOURCES = ["host_ffn.cpp"]
HEADERS = ["common.cuh", "kernels.h"]
LIB = os.path.join(HERE, "libmoe_b200.so")
LIB_DEBUG = os.path.join(HERE, "libmoe_b200_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def lib_path(debug: bool = False) -> str:
    return LIB_DEBUG if debug else LIB


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HOST_SOURCES + HEADERS]
    deps += [os.path.join(ROOT, "include", h) for h in ("moe.h", "moe_split.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    lib = lib_path(debug)
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(ROOT, "_build", "debug" if debug else "release")
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                    "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]
    if debug:
        flags += ["-DMOE_DEBUG_CHECKS"]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        subprocess.check_call([nvcc(), *flags, "-c", os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    for src in HOST_SOURCES:
        obj = os.path.join(objdir, src.replace(".cpp", ".o"))
        subprocess.check_call(["g++", "-O3", "-std=c++17", "-fPIC", "-fvisibility=hidden",
                               "-pthread", "-I", os.path.join(ROOT, "include"),
                               *(["-DMOE_DEBUG_CHECKS"] if debug else []),
                               "-c", os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    tmp = lib + f".{os.getpid()}.tmp"
    subprocess.check_call([nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static",
                           "-Xcompiler", "-pthread"])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv,
                debug="--debug-checks" in sys.argv))
