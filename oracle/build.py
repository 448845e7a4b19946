"""Builds the oracle's shared library (plain C, no GPU code).

Test infrastructure: only the test-suite, the smoke check and the benchmark's
CPU-baseline leg use the oracle.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "ep_oracle.c")
SRCS = [SRC, os.path.join(HERE, "ep_tile_ans.c")]


def build(force=False):
    """Compile ep_oracle.c and ep_tile_ans.c with strict IEEE double arithmetic (no contraction, no fast-math)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        [os.path.getmtime(f) for f in SRCS] + [os.path.getmtime(os.path.join(HERE, "ep_oracle.h"))]
    ):
        return LIB
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", LIB + ".tmp"] + SRCS + ["-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
