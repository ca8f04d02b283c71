"""Build the CPU oracle (test infrastructure) into oracle/liboracle.so with gcc.

Flags keep the arithmetic plain: no fast-math, no contraction of a*b+c into
fused multiply-adds, IEEE single precision for float (x86-64 SSE).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fno-fast-math",
          "-ffp-contract=off", "-fexcess-precision=standard", "-Wall", "-Wextra"]


def build(force=False):
    deps = [SRC, os.path.join(HERE, "oracle.h")]
    if (not force and os.path.exists(LIB)
            and all(os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps)):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
