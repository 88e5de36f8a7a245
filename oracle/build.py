"""Compile the float64 oracle (plain C) into oracle/liboracle_mla.so.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU-baseline leg
load the result.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mla_oracle.c")
LIB = os.path.join(HERE, "liboracle_mla.so")
# IEEE semantics: no fast-math, no contraction into fused multiply-adds
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(*sys.argv[1:2] or [SRC]))
