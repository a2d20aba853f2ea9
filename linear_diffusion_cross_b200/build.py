"""Build libfldce.so in-tree with nvcc for sm_100a.

    python -m linear_diffusion_cross_b200.build [--verbose]

The library is one CUDA translation unit (csrc/fldce_api.cu, which includes
the kernel headers) linked against the static CUDA runtime, so it carries no
dependency on the runtime PyTorch ships.  The output lands next to this file,
where the Python binding loads it from.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "fldce_api.cu")
DEPS = [os.path.join(PKG, "csrc", f) for f in ("ptx.cuh", "umma_gemm.cuh", "kernels.cuh")] + [
    os.path.join(ROOT, "include", "fldce.h")]
LIB = os.path.join(PKG, "libfldce.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC,-O2",
    "-cudart", "static",
    "-I" + os.path.join(ROOT, "include"),
]


def nvcc_path() -> str:
    p = shutil.which("nvcc")
    if p:
        return p
    p = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(p):
        return p
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfldce.so")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in [SRC, *DEPS, __file__])


def build(force: bool = False, verbose: bool = False, extra: tuple = ()) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    tmp = LIB + ".tmp"
    cmd += ["-o", tmp, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
