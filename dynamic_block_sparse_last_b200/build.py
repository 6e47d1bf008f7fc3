"""Compiles the CUDA library (csrc/) into _lib/libfpsparse.so for sm_100a.

Run as ``python -m dynamic_block_sparse_last_b200.build``; needs only nvcc
(cross-compiles without a GPU).
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(PKG, "csrc", f) for f in ("fp_sparse.cu", "fp_prefill.cpp")]
DEPS = SRCS + [os.path.join(PKG, "csrc", f) for f in ("ptx.cuh", "index_kernels.cuh", "attn_kernel.cuh",
                                                      "rope_pool.cuh", "share_kernels.cuh")] \
    + [os.path.join(ROOT, "include", f) for f in ("fp_sparse.h", "fp_prefill.h")]
LIB = os.path.join(PKG, "_lib", "libfpsparse.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc")


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    stale = force or not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if not stale:
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), *SRCS, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
