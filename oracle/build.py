"""Build the fp64 CPU oracle (test infrastructure) into oracle/liboracle.so.

Building the checker is not using it: the product library never links it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, "ecasq_oracle.cpp"), os.path.join(HERE, "ecasq_approx_oracle.cpp"),
        os.path.join(HERE, "ecasq_rans_oracle.cpp")]
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in SRCS):
        return LIB
    cmd = ["g++", "-O2", "-std=c++17", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", LIB] + SRCS
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
