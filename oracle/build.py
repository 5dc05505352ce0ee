"""Compile the C oracle into an in-tree shared library (test infrastructure).

gcc, C11, -O2 -fno-fast-math -ffp-contract=off: every float operation in the
oracle is one IEEE-754 binary32 operation rounded to nearest-even.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8bw_oracle.c")
HDR = os.path.join(HERE, "fp8bw_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
