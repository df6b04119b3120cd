"""Builds libgdla.so (sm_100a) in-tree with nvcc.

The library is one translation unit (csrc/gdla_lib.cu). cudart is linked
statically and the driver API is reached through cudaGetDriverEntryPoint, so
the .so loads on machines without a GPU driver (its calls then fail with
GDLA_ERR_CUDA).
"""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libgdla.so")
SOURCES = ["gdla_lib.cu", "gdla_api.cu", "gdla_prefill.cu", "gdla_prefill_bwd.cu", "gdla_prologue.cu", "gdla_decode.cu", "gdla_decode_noalloc.cu",
           "gdla_decode_latent.cu", "gdla_selftest.cu", "gdla_internal.h", "gdla_ptx.cuh", "gdla_prologue.h",
           "gdla_pair.cuh"]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the GDLA CUDA library cannot be built")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES] + [os.path.join(INCLUDE, "gdla.h"), __file__]
    return [f for f in files if os.path.exists(f)]


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/gdla_lib.cu into libgdla.so next to this file."""
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC, "-o", tmp,
           os.path.join(CSRC, "gdla_lib.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    # the compiler's intermediate files stay inside the repository
    scratch = os.path.join(os.path.dirname(PKG), "_build", "tmp")
    os.makedirs(scratch, exist_ok=True)
    subprocess.check_call(cmd, env={**os.environ, "TMPDIR": scratch})
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, verbose=True))
