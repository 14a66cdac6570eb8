"""Build the CPU oracle shared library (test infrastructure only).

Compiles ``janus_oracle.cpp`` into ``liboracle_janus.so`` next to it with
g++ -O2, OpenMP, and FP contraction off (so that a product and a sum are
rounded separately, as the source text says).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "janus_oracle.cpp")
LIB = os.path.join(HERE, "liboracle_janus.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off",
           "-shared", "-fPIC", SRC, "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
