"""Build libbs.so (the sm_100a decoder library) in place, next to this file.

    python lossless_entropy_coding_interleaved_b200/build.py [--verbose]

Run it as a script (or load it by path, as __graft_entry__.build does). Importing it
through the package would first load the library it is meant to rebuild.

nvcc cross-compiles for sm_100a without a GPU, so this runs on any host with CUDA 12.9.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libbs.so")
SOURCES = ["bs_kernels.cu", "bs_joint4.cu", "bs_encode_kernels.cu", "bs_noalloc.cu", "bs_fw.cu", "bs_fw_gemv.cu", "bs_fw_gemm.cu", "bs_plan.cpp", "bs_validate.cpp", "bs_encode.cpp",
           "bs_stream.cpp"]
HEADERS = ["bs_internal.h", "bs_device.cuh", "bs_host.h", "bs_fw.cuh", os.path.join(ROOT, "include", "bs.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
         "-Xcompiler", "-fPIC,-O2", "-shared", "-I", os.path.join(ROOT, "include")]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + [h if os.path.isabs(h) else os.path.join(CSRC, h)
                                                          for h in HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []),
           *[os.path.join(CSRC, s) for s in SOURCES], "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
