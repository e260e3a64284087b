"""Compile the fp64 CPU oracle into oracle/libhga_oracle.so (test infrastructure).

Plain gcc, -O2 without fast-math so that every sum keeps the order written in
hga_oracle.c; OpenMP only splits independent output rows across threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hga_oracle.c")
LIB = os.path.join(HERE, "libhga_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "hga_oracle.h"))
    ):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
