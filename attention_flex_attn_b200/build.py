"""Builds libflexattn.so in-tree for sm_100a with nvcc.

    python -m attention_flex_attn_b200.build [--verbose-ptxas]

The library links the CUDA runtime statically, so loading it needs no libcudart on
the library path; driver entry points (tensor-map encoding) are resolved at run time.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libflexattn.so")
OBJ_DIR = os.path.join(PKG, "_build")
# Translation units: the forward and backward kernels per (head dim, block mask), the
# persistent forward per head dim, the 8-bit forward, decode, and the C ABI.
# They compile in parallel and link into one shared library.
SOURCES = [os.path.join(CSRC, f) for f in (
    "flex_fwd_d128.cu", "flex_fwd_d128_blocks.cu", "flex_fwd_d64.cu", "flex_fwd_d64_blocks.cu",
    "flex_fwd_d128_persist.cu", "flex_fwd_d64_persist.cu",
    "flex_bwd_d128.cu", "flex_bwd_d64.cu", "flex_bwd_d128_blocks.cu", "flex_bwd_d64_blocks.cu", "flex_fwd_fp8.cu",
    "flex_decode_launch.cu", "flex_attn_api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(INCLUDE, "flex_attn.h")]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]
LINK_FLAGS = [*ARCH, "-shared", "-cudart", "static"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS + [os.path.abspath(__file__)])


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not stale():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(OBJ_DIR, os.path.splitext(os.path.basename(src))[0] + ".o")
        objs.append(obj)
        cmd = [nvcc(), *COMPILE_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
        procs.append((src, subprocess.Popen(cmd)))
    failed = [src for src, pr in procs if pr.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, "nvcc " + " ".join(os.path.basename(f) for f in failed))
    subprocess.check_call([nvcc(), *LINK_FLAGS, "-o", LIB + ".tmp", *objs])
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
