"""Build the CUDA library in-tree: ``python -m tiled_attention_22_b200.build``.

Compiles csrc/api.cu (which includes every kernel) with nvcc for sm_100a into
tiled_attention_22_b200/_lib/libtiled_attention.so.  No JIT cache is used: the
built file sits beside the sources so it travels with the repository.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_DIR = os.path.join(HERE, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libtiled_attention.so")
SOURCES = ["csrc/api.cu"]
DEPS = ["csrc/api.cu", "csrc/attn_fwd_kernels.cuh", "csrc/attn_fwd_persistent.cuh", "csrc/attn_fwd_launch.cuh", "csrc/tma_host.cuh",
        "csrc/decode_kernels.cuh", "csrc/decode_launch.cuh", "csrc/merge_kernels.cuh", "csrc/prepass_kernels.cuh", "csrc/ptx.cuh",
        "../include/tiled_attention.h"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(os.path.join(HERE, d)) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    os.makedirs(LIB_DIR, exist_ok=True)
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(HERE, "csrc"), "-o", LIB_PATH + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(HERE, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
