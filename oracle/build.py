"""Build the CPU oracle library (liboracle.so) with gcc.

The oracle is test infrastructure: a plain C reference of the AB-Attention
hot path.  It is compiled without fused-multiply-add contraction so that its
fp32 k-means arithmetic is exactly the sequence the source spells out.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "absa_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "absa_oracle.h"))
    ):
        return LIB
    cmd = [
        "gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
        "-fopenmp", "-shared", "-fPIC", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
