"""Build the CPU oracle (plain C, f64) into oracle/libcoli_oracle.so.

Test infrastructure: compiled so that the tests, the smoke check and the
benchmark's CPU-baseline leg can call it.  Nothing in the product path loads it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "coli_oracle.c")
LIB = os.path.join(HERE, "libcoli_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "coli_oracle.h"))):
        return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
