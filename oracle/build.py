"""Compile the CPU oracle into ``oracle/libtq_oracle.so``.

Test infrastructure: the tests, the smoke check and the benchmark's CPU-baseline
leg load the result; the product library never does.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tq_oracle.cpp")
LIB = os.path.join(HERE, "libtq_oracle.so")

# No FMA contraction and no fast-math: every binary32 step is one IEEE operation.
CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build_oracle(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["g++", *CXXFLAGS, "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force=True))
