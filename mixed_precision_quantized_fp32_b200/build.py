"""Build the CUDA library (sm_100a) in-tree: mixed_precision_quantized_fp32_b200/libmoe_b200.so.

nvcc cross-compiles without a GPU.  No fast-math: the packing kernels rely on
IEEE division and round-half-even.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_b200.so")
BUILD = os.path.join(HERE, "_build")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]

GEN_SRC = os.path.join(ROOT, "gen", "gen_device.cu")
GEN_LIB = os.path.join(ROOT, "gen", "libmoegen.so")
GEN_HOST_SRC = os.path.join(ROOT, "gen", "gen_host.c")
GEN_HOST_LIB = os.path.join(ROOT, "gen", "libmoegen_host.so")


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(ROOT, "include", "moe.h")]
    objs = []
    for s in srcs:
        o = os.path.join(BUILD, os.path.basename(s) + ".o")
        objs.append(o)
        if force or _stale(o, [s] + hdrs):
            cmd = [NVCC, *ARCH, *FLAGS, "-c", s, "-o", o]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            subprocess.run(cmd, check=True)
    if force or _stale(LIB, objs):
        subprocess.run([NVCC, *ARCH, "-shared", *objs, "-o", LIB + ".tmp", "-lcudart"], check=True)
        os.replace(LIB + ".tmp", LIB)
    if force or _stale(GEN_LIB, [GEN_SRC]):
        subprocess.run([NVCC, *ARCH, *FLAGS, "-shared", GEN_SRC, "-o", GEN_LIB + ".tmp"], check=True)
        os.replace(GEN_LIB + ".tmp", GEN_LIB)
    build_gen_host(force)
    return LIB


def build_gen_host(force: bool = False) -> str:
    """The generator's multi-threaded host fill (plain C); test and bench infrastructure."""
    if force or _stale(GEN_HOST_LIB, [GEN_HOST_SRC]):
        subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                        "-fvisibility=hidden", GEN_HOST_SRC, "-o", GEN_HOST_LIB + ".tmp"], check=True)
        os.replace(GEN_HOST_LIB + ".tmp", GEN_HOST_LIB)
    return GEN_HOST_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
