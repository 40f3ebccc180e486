"""Build the CUDA library libqlin.so in-tree with nvcc for sm_100a.

Every translation unit under csrc/ is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` (no fast-math: the
quantisers and epilogues rely on IEEE division and separately rounded
multiplies) and linked into one shared library with the CUDA runtime linked
statically, so the library loads on a machine without a GPU driver (it then
reports QLIN_ERR_NO_DEVICE at run time).
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libqlin.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr"]
SOURCES = ["quantize.cu", "quantize_bs.cu", "gemm.cu", "api.cu", "noalloc.cu", "moe.cu"]
HEADERS = ["ptx.cuh", "internal.h", "pdl.cuh", "quant_math.cuh"]


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False, extra: list[str] | None = None) -> str:
    os.makedirs(BUILD, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "qlin.h")]
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if force or _stale(o, [s, *hdrs, __file__]):
            jobs.append([NVCC, *ARCH, *FLAGS, *(extra or []), "-c", s, "-o", o])

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr)

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        list(ex.map(run, jobs))
    if jobs or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        run([NVCC, *ARCH, "-shared", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    return LIB




SWEEP_SRC = os.path.join(HERE, "sweep", "qlin_sweep.cu")
SWEEP_BIN = os.path.join(HERE, "qlin_sweep")


def build_sweep(verbose: bool = False) -> str:
    """Build the offline dispatch-table sweep (links libqlin.so through the C ABI)."""
    lib = build(verbose=verbose)
    if not os.path.exists(SWEEP_BIN) or _stale(SWEEP_BIN, [SWEEP_SRC, lib, os.path.join(INCLUDE, "qlin.h")]):
        cmd = [NVCC, *ARCH, "-O2", "-std=c++17", "-I", INCLUDE, SWEEP_SRC, "-o", SWEEP_BIN, "-L", HERE, "-lqlin",
               "-Xlinker", "-rpath,$ORIGIN"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return SWEEP_BIN


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force="-f" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
    if "--sweep" in sys.argv:
        print(build_sweep(verbose="-v" in sys.argv))
