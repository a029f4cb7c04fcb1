"""Build step for the CUDA library: nvcc, sm_100a only, in-tree output.

``python -m gemm_epilogues_tcgen05_b200.build`` (or ``build()``) compiles the
translation units under ``csrc/`` -- the host side (``gemm_epi.cu``) and the
kernel instances (``inst_*.cu``) -- in parallel into objects under
``_build/``, then links them into ``libgemm_epi.so`` next to this file. The
CUDA runtime is linked statically and the driver is reached through
``cudaGetDriverEntryPoint``, so the library loads on a machine without a GPU
(every compute call then fails with an error code).
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libgemm_epi.so")
CSRC = os.path.join(HERE, "csrc")
OBJ_DIR = os.path.join(HERE, "_build")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = os.path.join(cuda, "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def units() -> list[str]:
    """The translation units, largest (most kernel instances) first."""
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    order = ("inst_skinny", "inst_tile", "inst_pair", "gemm_epi")
    return sorted(srcs, key=lambda s: next((i for i, p in enumerate(order) if os.path.basename(s).startswith(p)), 9))


def compile_command(src: str, obj: str, verbose_ptxas: bool = False) -> list[str]:
    cmd = [_nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler",
           "-fvisibility=hidden", "-I", INCLUDE, "-c", "-o", obj, src]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def link_command(objs: list[str], out: str) -> list[str]:
    return [_nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", out, *objs]


def _headers() -> list[str]:
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
            glob.glob(os.path.join(INCLUDE, "*.h")))


def _sources() -> list[str]:
    return units() + _headers()


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int | None = None) -> str:
    if not force and not needs_build():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    todo, objs = [], []
    for src in units():
        obj = os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header):
            todo.append((src, obj))
    jobs = jobs or max(1, min(len(todo), os.cpu_count() or 1))

    def run(pair):
        src, obj = pair
        tmp = obj + f".tmp{os.getpid()}"
        subprocess.check_call(compile_command(src, tmp, verbose_ptxas))
        os.replace(tmp, obj)

    with concurrent.futures.ThreadPoolExecutor(max_workers=jobs) as ex:
        for f in [ex.submit(run, t) for t in todo]:
            f.result()
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(link_command(objs, tmp))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
