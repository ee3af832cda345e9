"""Build libtriattn.so in-tree for sm_100a (nvcc cross-compiles; no GPU needed).

    python -m triangle_attention_biomolecular_b200.build [--force]

The library is csrc/api.cu (which includes the kernels) plus csrc/bwd_static.cu,
compiled with ``-gencode arch=compute_100a,code=sm_100a`` and the CUDA
runtime linked statically, so it loads on a machine without a GPU driver and
depends on nothing but libc/libstdc++ at load time.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
LIB = os.path.join(_HERE, "libtriattn.so")
SRC = os.path.join(_HERE, "csrc", "api.cu")
# the backward on a static scratch array: a translation unit (module) of its own
SRC_STATIC = os.path.join(_HERE, "csrc", "bwd_static.cu")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(_HERE, "csrc", "*"))) + [os.path.join(_ROOT, "include", "tri_attn.h")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-Xptxas", "-v" if verbose else "-O3",
           SRC, SRC_STATIC, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose:
        print(r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
