"""Build the CUDA library ``libnomas.so`` in-tree with nvcc for sm_100a.

The library links the CUDA runtime statically, so loading it needs no GPU
and no driver; the driver is reached at the first CUDA call.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["nomas_host.cu", "rope_commit.cu", "seg_attn.cu", "camera_attn.cu", "nomas_static.cu",
           "nomas_selftest.cu"]
HEADERS = ["nomas_internal.h", "nomas_ptx.cuh", "nomas_f16.cuh", "nomas_div127.cuh"]
LIB = os.path.join(HERE, "libnomas.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "nomas.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
           "-I" + os.path.join(ROOT, "include"), "-o", tmp]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += list(extra or [])
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
