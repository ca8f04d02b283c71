"""Build libmxq.so (the sm_100a CUDA library) in-tree with nvcc.

The library is one translation unit (csrc/mxq.cu includes every kernel) so
that the device status word is a single symbol without relocatable device
code. The CUDA runtime is linked statically; the stream handles passed in by
PyTorch are driver objects and work across runtimes.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmxq.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC,-O2",
         "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
         "-cudart", "static", "--expt-relaxed-constexpr"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)) + [os.path.join(INCLUDE, "mxq.h")]


def build(force=False, verbose=False, extra=()):
    srcs = sources()
    if (not force and os.path.exists(LIB)
            and all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in srcs)):
        return LIB
    cmd = [NVCC, *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, *extra,
           os.path.join(CSRC, "mxq.cu"), "-o", LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "-v" in sys.argv else []
    print(build(force=True, verbose=True, extra=extra))
