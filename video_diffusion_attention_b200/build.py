"""Build libtara_attn.so in-tree with nvcc for sm_100a.

    python -m video_diffusion_attention_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libtara_attn.so")
# the same sources with the kernels' device-side checks compiled in (-DTARA_DEBUG=1)
LIB_DEBUG = os.path.join(LIB_DIR, "libtara_attn_debug.so")
SOURCES = [os.path.join(CSRC, "tara_abi.cu"), os.path.join(CSRC, "tara_pack.cpp"),
           os.path.join(CSRC, "tara_host.cpp")]
HEADERS = [os.path.join(ROOT, "include", "tara_attn.h")] + [
    os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cuh", ".h"))]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    """Compile the release library (or, with debug=True, libtara_attn_debug.so with the
    kernels' device-side checks) if a source is newer than it or force is set."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not stale(lib):
        return lib
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc()] + NVCC_FLAGS + ["-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if debug:
        cmd += ["-DTARA_DEBUG=1"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", tmp] + SOURCES
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv,
                debug="--debug" in sys.argv))
