"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so.

gcc with -O2 -ffp-contract=off and no fast-math: every float operation stays a
single IEEE binary32 (or binary64) operation rounded to nearest-even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra"]


def build(src=SRC, out=LIB, extra=()):
    """Compile `src` to the shared library `out`; returns `out`."""
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def needs_build(out=LIB, src=SRC):
    hdr = os.path.join(HERE, "oracle.h")
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return t < os.path.getmtime(src) or t < os.path.getmtime(hdr)


if __name__ == "__main__":
    print(build(*sys.argv[1:2]) if len(sys.argv) > 1 else build())
