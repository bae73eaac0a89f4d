"""Build the CUDA library ``libkda_b200.so`` in-tree for sm_100a.

One translation unit (``csrc/kda_api.cu``) holds every kernel and the C ABI
declared in ``include/kda.h``.  The result is a plain shared library with an
extern "C" interface; Python binds it through ctypes.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkda_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared",
         "-I" + os.path.join(ROOT, "include")]


def sources():
    return [os.path.join(SRC_DIR, f) for f in sorted(os.listdir(SRC_DIR))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(ROOT, "include", "kda.h")]


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = [NVCC, *FLAGS, *extra, "-o", LIB, os.path.join(SRC_DIR, "kda_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
