"""Compile the CPU oracle (ep_oracle.cpp) into oracle/liboracle.so.

Test infrastructure only: the oracle is the checker the tests, the smoke check
and the benchmark's CPU-baseline leg compare against.  Plain g++, no CUDA.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [
        "g++", "-std=c++17", "-O2", "-fPIC", "-shared",
        # fp64 sums stay in program order: no contraction, no reassociation.
        "-ffp-contract=off", "-fno-fast-math",
        SRC, "-o", LIB + ".tmp",
    ]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
