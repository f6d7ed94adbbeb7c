"""Builds libfa.so (the sm_100a kernel and its C ABI) in-tree with nvcc.

Usage: python -m tiled_online_softmax_03_b200.build [--verbose]
"""

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fa_fwd_sm100.cu")
DEPS = [SRC, os.path.join(PKG, "csrc", "fa_ptx.cuh"), os.path.join(PKG, "csrc", "fa_schedule.cuh"),
        os.path.join(PKG, "csrc", "fa_bwd_sm100.cuh"),
        os.path.join(PKG, "csrc", "fa_host_pipeline.cuh"),
        os.path.join(PKG, "csrc", "fa_host.cuh"),
        os.path.join(ROOT, "include", "fa.h")]
LIB = os.path.join(PKG, "libfa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc():
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force=False, verbose=False):
    """Compile libfa.so unless it is newer than every source. Returns its path."""
    if not force and up_to_date():
        return LIB
    cmd = [nvcc()] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
        ["-o", LIB, SRC, "-lcudart"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libfa.so")
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
