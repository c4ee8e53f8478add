"""Build libdq.so (the C-ABI of include/dq.h) in-tree with nvcc for sm_100a,
and libdq_checked.so: the same sources compiled with DQ_CHECKED, whose
attention kernels also count containers decoded past their bytes
(dq_stats.overreads). Select the checked library with DQ_LIBRARY=<path>.

Usage: python -m decode_attention_dq_b200.build [--force] [--verbose] [--checked]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "lib", "libdq.so")
LIB_CHECKED = os.path.join(HERE, "lib", "libdq_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "--expt-relaxed-constexpr",
    "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        [os.path.join(INCLUDE, "dq.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.exists(cand) or cand == "nvcc"):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not (force or needs_build(lib)):
        return lib
    os.makedirs(os.path.dirname(lib), exist_ok=True)
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DDQ_CHECKED"] if checked else []), "-shared", "-I", INCLUDE, "-I", CSRC,
           *sources(), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas")
        cmd.insert(2, "-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
