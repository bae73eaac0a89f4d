"""Compile the fp64 CPU oracle (test infrastructure only) into a shared library.

The oracle is plain C built with ``-O2`` and no fast-math flags, so its
arithmetic is IEEE fp64 in the order written in ``kda_oracle.c``.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
LIB = os.path.join(HERE, "libkda_oracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Build ``out`` from ``src`` unless it is already newer than the source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-std=c11", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
