"""Build the CUDA library libbitnet_b200.so in-tree (sm_100a only).

One translation unit (csrc/bitnet.cu) compiled by nvcc for
arch=compute_100a,code=sm_100a, linked against the shared CUDA runtime so the
library and PyTorch use one runtime instance (same current device, streams).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libbitnet_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    out = [os.path.join(INCLUDE, "bitnet.h")]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, f))
    return out


def nvcc_cmd(out, extra=()):
    return [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-shared", "-Xcompiler", "-fPIC", "-cudart", "shared",
            "-Xlinker", "-rpath=/usr/local/cuda/lib64",
            "-I", INCLUDE, "-I", CSRC, *extra, "-o", out, os.path.join(CSRC, "bitnet.cu")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in sources()):
            return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    extra = ["-Xptxas", "-v"] if verbose else []
    subprocess.check_call(nvcc_cmd(tmp, extra))
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
