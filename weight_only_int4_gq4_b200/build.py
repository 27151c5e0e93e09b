"""Build libgq4.so in-tree with nvcc for sm_100a (B200).  Cross-compiles without a GPU."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "gq4_host.cu")
LIB = os.path.join(HERE, "libgq4.so")
LIB_CHECKED = os.path.join(HERE, "libgq4_checked.so")  # -DGQ4_CHECKED: bounds-checked kernels
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
         "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc")]


def sources():
    d = os.path.join(HERE, "csrc")
    return [os.path.join(d, f) for f in os.listdir(d)] + [os.path.join(ROOT, "include", "gq4.h")]


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile libgq4.so (or, with checked, libgq4_checked.so with GQ4_CHECKED defined)."""
    lib = LIB_CHECKED if checked else LIB
    newest = max(os.path.getmtime(f) for f in sources())
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-DGQ4_CHECKED"] if checked else []), SRC, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
