"""Builds libsga.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsga.so")
LIB_DEBUG = os.path.join(PKG, "libsga_debug.so")  # SGA_DEBUG: device invariant checks
SOURCES = ["sga_api.cu", "sga_index.cu", "sga_topk.cu", "sga_attend.cu", "sga_gemm.cu", "sga_layer.cu",
           "sga_warmup.cu", "sga_diag.cu"]
DEPS = SOURCES + ["sga_ptx.cuh", "sga_internal.cuh", "sga_host.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsga")
    return cand


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in DEPS] + [os.path.join(ROOT, "include", "sga.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every kernel source into one shared library next to this file.
    With `debug`, libsga_debug.so: the same code with the SGA_DEBUG invariant
    checks compiled in (a failed check records SGA_ERR_INTERNAL; nothing traps)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc_path(), "-std=c++17", "-O3", *ARCH, "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           *(["-DSGA_DEBUG"] if debug else []), *[os.path.join(CSRC, f) for f in SOURCES], "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
