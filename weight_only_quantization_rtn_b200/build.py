"""Build the W4A16 CUDA library in-tree: libw4a16.so next to this file.

    python -m weight_only_quantization_rtn_b200.build [--verbose]

nvcc compiles the translation units csrc/w4a16.cu (INT4) and csrc/w8a16.cu
(8-bit codes) into one library for sm_100a only
(-gencode arch=compute_100a,code=sm_100a), without fast-math (the quantizer's
division and rounding must be IEEE), with -lineinfo for profiling.  The CUDA
runtime is linked statically, so the library needs only the driver at run time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libw4a16.so")
SRCS = [os.path.join(HERE, "csrc", "w4a16.cu"), os.path.join(HERE, "csrc", "w8a16.cu")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
         "--expt-relaxed-constexpr", "-cudart", "static", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the W4A16 CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*")) +
                  [os.path.join(ROOT, "include", "w4a16.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *FLAGS, "-o", tmp, *SRCS]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose, verbose=a.verbose))
    sys.exit(0)
