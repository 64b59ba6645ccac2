"""Compile the CPU oracle (oracle/hbl_oracle.c) into oracle/liboracle.so.

Test infrastructure: the oracle is built so that tests, the smoke check and the
benchmark's CPU baseline can call it.  The CUDA library never links it.

Flags: -O2 with floating-point contraction off, so that every fp32 operation
in the C source is one IEEE-rounded operation (no fused multiply-add).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hbl_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
