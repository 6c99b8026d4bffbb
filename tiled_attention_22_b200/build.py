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


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Build the library.  ``defines`` ("NAME=VALUE" strings) select compile-time variants of the
    kernels (the measurement variants named in the kernel sources); a variant build goes to
    ``out`` and never replaces the in-tree library."""
    target = out or LIB_PATH
    if not force and not defines and out is None and up_to_date():
        return LIB_PATH
    os.makedirs(os.path.dirname(os.path.abspath(target)), exist_ok=True)
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(HERE, "csrc"), "-o", target + ".tmp"]
    cmd += [f"-D{d}" for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(HERE, s) for s in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(target + ".tmp", target)
    return target


if __name__ == "__main__":
    import argparse

    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", action="store_true", help="ptxas register / spill report")
    ap.add_argument("--define", action="append", default=[], help="NAME=VALUE for a kernel variant (repeatable)")
    ap.add_argument("--out", default=None, help="output path for a variant build")
    a = ap.parse_args()
    if a.define and not a.out:
        ap.error("a variant build (--define) needs --out")
    print(build(force=a.force, verbose=a.v, defines=a.define, out=a.out))
