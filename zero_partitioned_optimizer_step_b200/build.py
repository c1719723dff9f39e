"""Build libzero.so in-tree: the planner (C++) and the sm_100a kernels (CUDA).

    python -m zero_partitioned_optimizer_step_b200.build [--force] [--verbose]

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked
statically, so the library loads on a machine without a driver (queries and
argument checks work there; launches return ZERO_ECUDA).
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libzero.so")
SOURCES = [os.path.join(CSRC, f) for f in ("zero_plan.cpp", "zero_step.cu", "zero_noalloc.cu", "zero_peer.cu", "zero_reshard.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("zero_internal.h", "zero_device.cuh", "zero_tma.cuh",
                                             "zero_guard.cuh", "zero_host.cuh", "zero_ring.cuh",
                                             "zero_trace.h")] + \
    [os.path.join(ROOT, "include", "zero.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-fmad=false",               # no FMA contraction in the Adam arithmetic
    "-Xcompiler", "-fPIC,-fvisibility=hidden,-ffp-contract=off",
    "-cudart", "static",
    "-shared",
]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS + [__file__])


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += SOURCES + ["-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
