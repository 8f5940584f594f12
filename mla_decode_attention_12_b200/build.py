"""Builds the C-ABI shared library ``_mla_decode.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m mla_decode_attention_12_b200.build`` (or call :func:`build`).
The CUDA runtime is linked statically, so the library needs only the NVIDIA
driver at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "_mla_decode.so")
SOURCES = [os.path.join(CSRC, "mla_decode.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "scheduler.cuh")] + [
    os.path.join(ROOT, "include", "mla_decode.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def up_to_date(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    """Compile the library if any source is newer than it; returns its path.

    ``extra`` adds nvcc flags and ``out`` names another file: instrumented or test-only
    builds of the same sources (``-DMLA_TIMELINE``, ``-DMLA_TEST_WITHHOLD_K_PAGE=n``) go
    to their own files, never to the product library's."""
    if not force and up_to_date(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", tmp, *SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
