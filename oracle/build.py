"""Compile the fp64 CPU oracle (``fa_oracle.c``) into ``liboracle.so`` beside this file.

Test infrastructure only: the CUDA library never uses the oracle. ``build(src, out)`` also serves the
tests that compile deliberately broken copies of the oracle source into a temporary directory.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fa_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(src=SRC, out=LIB, quiet=True):
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-o", out, src, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if not quiet:
        print(" ".join(cmd))
    return out


def ensure_built():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        build()
    return LIB


if __name__ == "__main__":
    build(quiet=False)
    sys.exit(0)
