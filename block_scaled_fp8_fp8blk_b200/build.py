"""In-tree build of the package's native libraries.

* ``libfp8blk.so``       -- the CUDA kernels and the C ABI (``include/fp8blk.h``),
  compiled for sm_100a only;
* ``libfp8blk_synth.so`` -- the seeded input generator (plain C).

Run ``python -m block_scaled_fp8_fp8blk_b200.build`` (``--force`` rebuilds).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfp8blk.so")
SYNTH_SRC = os.path.join(PKG, "synth.c")
SYNTH_LIB = os.path.join(PKG, "libfp8blk_synth.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = [os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]
    for c in cand:
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(out: str, srcs) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in srcs)


def build_synth(force: bool = False) -> str:
    if force or _stale(SYNTH_LIB, [SYNTH_SRC]):
        tmp = SYNTH_LIB + f".tmp{os.getpid()}"
        subprocess.run([os.environ.get("CC", "gcc"), "-O2", "-fPIC", "-shared", "-pthread",
                        SYNTH_SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, SYNTH_LIB)
    return SYNTH_LIB


def cuda_sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def build_cuda(force: bool = False, verbose_ptxas: bool = False) -> str:
    srcs = cuda_sources()
    deps = srcs + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    if not srcs:
        raise RuntimeError("no CUDA sources found")
    if not (force or _stale(LIB, deps)):
        return LIB
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s) + ".o")
        subprocess.run([nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", s, "-o", o],
                       check=True)
        objs.append(o)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs,
                    "-o", tmp, "-lcudart"], check=True)
    os.replace(tmp, LIB)
    return LIB


def build(force: bool = False) -> None:
    build_synth(force)
    build_cuda(force)


if __name__ == "__main__":
    build(force="--force" in sys.argv)
    print(LIB)
