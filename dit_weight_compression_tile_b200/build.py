"""Builds libeptile.so in-tree: the sm_100a decode kernel and the host compressor/parser.

nvcc compiles the CUDA source for sm_100a only; host C++ is compiled with strict IEEE
double arithmetic (no contraction) because the encoder's rounding decisions are part of
the stream format.
"""
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libeptile.so")
SOURCES = ["decode.cu", "linear.cu", "device_encode.cu", "host_encode.cpp", "host_stream.cpp", "tile_ans.cu",
           "tile_ans_host.cpp"]
HEADERS = [os.path.join(CSRC, h) for h in ("format.h", "encode_math.h", "encode_host.h", "device_util.cuh",
                                           "decode_core.cuh", "tile_ans.h")] + \
    [os.path.join(ROOT, "include", "eptile.h")]


def nvcc():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libeptile.so")
    return cand


def build(force=False, verbose=False):
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(f) for f in srcs + HEADERS)
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", "-shared", "-lineinfo",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC,-O2,-ffp-contract=off,-fno-fast-math,-pthread",
           "-o", LIB + ".tmp"] + srcs + ["-lpthread"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose="-v" in sys.argv))
