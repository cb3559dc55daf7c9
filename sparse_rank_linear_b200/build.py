"""Build the SALR CUDA library in-tree: ``python -m sparse_rank_linear_b200.build``.

Produces ``sparse_rank_linear_b200/libsalr.so`` for sm_100a (B200) with nvcc.  No GPU is
needed to build.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsalr.so")
SOURCES = ["salr_api.cu"]
HEADERS = ["sm100.cuh", "salr_block.cuh", "salr_decode.cuh", "salr_codec.cuh", "salr_prefill.cuh",
           "salr_stream.cuh", "salr_svd.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=()) -> list:
    return [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
            "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), *extra,
            *[os.path.join(CSRC, s) for s in SOURCES], "-o", out, "-cudart", "static"]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "salr.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


# Debug build: every data-derived offset in the kernels is checked; a failed check sets
# the range bit of the handle's status word (salr_sync_status then reports an error)
# instead of touching memory out of bounds.  Load it with SALR_LIBRARY=<this path>.
LIB_CHECKS = os.path.join(HERE, "libsalr_checks.so")


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    out = LIB_CHECKS if checks else LIB
    if force or stale(out):
        cmd = command(out, ("-DSALR_CHECKS",) if checks else ())
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, checks="--checks" in sys.argv)
