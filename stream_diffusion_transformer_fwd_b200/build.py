"""Build libig4.so (the CUDA library behind include/ig4.h) in-tree with nvcc.

    python -m stream_diffusion_transformer_fwd_b200.build [--verbose-ptxas]

Compiles for sm_100a only; needs no GPU (nvcc cross-compiles).  The shared
library lands next to this file, where the Python binding loads it.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libig4.so")
SOURCES = ["ig4_api.cu"]
DEPS = ["ig4_api.cu", "ig4_ptx.cuh", "ig4_gemm.cuh", "ig4_attention.cuh", "ig4_small.cuh",
        "ig4_mx8.cuh",
        "ig4_nvf4.cuh", "ig4_parallel.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "ig4.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [
        nvcc_path(), "-O3", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
        "-I", INCLUDE, "-I", CSRC,
        "-o", LIB + ".tmp",
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    path = build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(path)
