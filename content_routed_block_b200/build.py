"""Build libssa.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m content_routed_block_b200.build [--verbose]

The CUDA runtime is linked statically, so the library has no dependency on a
GPU driver at load time (the driver is reached at first use).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "ssa.cu")
OUT = os.path.join(HERE, "libssa.so")
DEPS = [os.path.join(HERE, "csrc", f) for f in
        ("ssa.cu", "common.cuh", "pool.cuh", "route.cuh", "route_tc.cuh", "consensus.cuh",
         "cumulant.cuh", "decode.cuh", "tree.cuh", "backward.cuh", "backward_tc.cuh",
         "attend.cuh")] + \
       [os.path.join(ROOT, "include", "ssa.h")]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    p = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(p):
        return p
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return OUT
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
           "-I", os.path.join(ROOT, "include"), "-o", OUT + ".tmp", SRC, *extra]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(OUT)
