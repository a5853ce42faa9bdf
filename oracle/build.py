"""Build the CPU oracle shared library (test infrastructure only).

Compiles ``fg8_oracle.cpp`` into ``liboracle.so`` beside it with strict IEEE
floating point (no fast-math, no FMA contraction) and OpenMP over rows.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fg8_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")


def compile_library(src: str, out: str) -> str:
    """Compile one oracle source file into a shared library at `out`."""
    cmd = ["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", src, "-o", out]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    compile_library(SRC, LIB + ".tmp")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
