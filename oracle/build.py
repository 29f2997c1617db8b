"""Build the fp64 CPU oracle into oracle/libgrinqh_oracle.so.

The oracle is test infrastructure: only the tests, the package smoke check and
the benchmark's CPU-baseline leg load it. Compiled without fast-math and without
floating-point contraction so that every fp64 operation rounds exactly as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "grinqh_oracle.cpp")
LIB = os.path.join(HERE, "libgrinqh_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", SRC, "-o", LIB + ".tmp"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
