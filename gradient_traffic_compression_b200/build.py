"""Build libtlc.so (the C ABI of include/tlc.h) in-tree with nvcc for sm_100a.

The arithmetic must match a plain sequential IEEE fp32 implementation bit for
bit, so the device code is compiled without FMA contraction (-fmad=false),
with IEEE division and square root, and without flush-to-zero.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SOURCES = ["tlc_api.cu", "tlc_compress.cu", "tlc_decode.cu", "tlc_noalloc.cu"]
HEADERS = ["tlc_device.cuh", "tlc_internal.h"]
LIB_NAME = "libtlc.so"
DEBUG_LIB_NAME = "libtlc_debug.so"   # -DTLC_DEBUG: recording bounds checks, canaries

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def library_path(debug: bool = False) -> str:
    return os.path.join(PKG, DEBUG_LIB_NAME if debug else LIB_NAME)


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libtlc.so")


def _inputs():
    yield os.path.join(ROOT, "include", "tlc.h")
    for f in SOURCES + HEADERS:
        yield os.path.join(CSRC, f)


def is_stale(debug: bool = False) -> bool:
    lib = library_path(debug)
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build_library(verbose: bool = False, ptxas_info: bool = False, debug: bool = False) -> str:
    """Compile every CUDA source into libtlc.so next to this file (debug:
    libtlc_debug.so, with -DTLC_DEBUG)."""
    out = library_path(debug)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(["-DTLC_DEBUG"] if debug else []), "-o", tmp,
           *[os.path.join(CSRC, f) for f in SOURCES]]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


KERNEL_SOURCES = {
    "k_absmax": ["tlc_compress.cu", "tlc_device.cuh", "tlc_internal.h"],
    "k_quant_zre": ["tlc_compress.cu", "tlc_device.cuh", "tlc_internal.h"],
    "k_zre_place": ["tlc_compress.cu", "tlc_device.cuh", "tlc_internal.h"],
    "k_decode_write": ["tlc_decode.cu", "tlc_device.cuh", "tlc_internal.h"],
    "k_decode_accumulate": ["tlc_decode.cu", "tlc_device.cuh", "tlc_internal.h"],
    "k_decode_count": ["tlc_decode.cu", "tlc_device.cuh", "tlc_internal.h"],
}


def source_digest(kernel: str | None = None) -> str:
    """Short SHA-256 over the compiler flags and the sources of one kernel
    (or of the whole library); identifies which build a stored profile
    belongs to."""
    import hashlib
    h = hashlib.sha256(" ".join(NVCC_FLAGS).encode())
    paths = ([os.path.join(CSRC, f) for f in KERNEL_SOURCES[kernel]] if kernel
             else list(_inputs()))
    for p in paths:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode() + b"\0" + f.read())
    return h.hexdigest()[:12]


def ensure_built(debug: bool = False) -> str:
    if is_stale(debug):
        build_library(debug=debug)
    return library_path(debug)


if __name__ == "__main__":
    print(build_library(verbose=True, ptxas_info="-v" in sys.argv, debug="--debug" in sys.argv))
