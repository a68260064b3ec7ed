"""Build libwd.so (sm_100a) in-tree with nvcc.

    python -m flow_matching_video_b200.build [--verbose]

The library is a single translation unit (csrc/wd_lib.cu) compiled for
sm_100a only; the result lands next to this file so that it travels with the
source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libwd.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(SRC, f) for f in os.listdir(SRC) if f.endswith((".cu", ".cuh"))) + [
        os.path.join(HERE, "..", "include", "wd.h")]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    # a temporary name per process, renamed into place atomically: ranks that
    # start together never write into one file, and a loader never sees half a file
    tmp = f"{OUT}.{os.getpid()}.tmp"
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "-o", tmp, os.path.join(SRC, "wd_lib.cu")]
    # compile-time options of the kernels, e.g. WD_NVCC_DEFINES="WD_ATTN_SELF_BK=64"
    cmd += ["-D" + d for d in os.environ.get("WD_NVCC_DEFINES", "").split()]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libwd.so")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(OUT)
