"""Builds libsparse_attn.so in-tree with nvcc for sm_100a (no GPU needed), and
its profiling variant libsparse_attn_trace.so (the same sources with
-DSA_TRACE: per-CTA phase marks for device timelines)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsparse_attn.so")
LIB_TRACE = os.path.join(HERE, "libsparse_attn_trace.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def sources():
    return sorted(os.path.join(SRC_DIR, f) for f in os.listdir(SRC_DIR) if f.endswith((".cu", ".cuh")))


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    out = LIB_TRACE if trace else LIB
    deps = sources() + [os.path.join(INCLUDE, "sparse_attn.h")]
    if not force and os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(d) for d in deps):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = out + f".{os.getpid()}.tmp"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DSA_TRACE"] if trace else []), "-o", tmp, os.path.join(SRC_DIR, "sparse_attn.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, trace="--trace" in sys.argv))
