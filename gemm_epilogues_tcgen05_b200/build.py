"""Build step for the CUDA library: one nvcc call, sm_100a only, in-tree output.

``python -m gemm_epilogues_tcgen05_b200.build`` (or ``build()``) compiles
``csrc/gemm_epi.cu`` into ``libgemm_epi.so`` next to this file. The CUDA
runtime is linked statically and the driver is reached through
``cudaGetDriverEntryPoint``, so the library loads on a machine without a GPU
(every compute call then fails with an error code).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libgemm_epi.so")
SRC = os.path.join(HERE, "csrc", "gemm_epi.cu")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(cuda, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def nvcc_command(out: str, verbose_ptxas: bool = False) -> list[str]:
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared", "-cudart", "static",
           "-I", INCLUDE, "-o", out, SRC]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def _sources() -> list[str]:
    return glob.glob(os.path.join(HERE, "csrc", "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(nvcc_command(tmp, verbose_ptxas))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
