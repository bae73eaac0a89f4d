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
DEBUG_LIB = os.path.join(HERE, "libkda_b200_debug.so")   # device-side bounds checks
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared",
         "-I" + os.path.join(ROOT, "include")]


def sources():
    return [os.path.join(SRC_DIR, f) for f in sorted(os.listdir(SRC_DIR))
            if f.endswith((".cu", ".cuh"))] + [os.path.join(ROOT, "include", "kda.h")]


def _build_one(out, extra, force, verbose):
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    cmd = [NVCC, *FLAGS, *extra, "-o", out, os.path.join(SRC_DIR, "kda_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Build the release library (returned) and, unless extra flags are given, the
    debug-checked one beside it."""
    if not extra:
        _build_one(DEBUG_LIB, ["-DKDA_DEBUG=1"], force, False)
    return _build_one(LIB, list(extra), force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
