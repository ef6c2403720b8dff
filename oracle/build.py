"""Build the oracle's shared library (plain C, fp64) with gcc.

TEST INFRASTRUCTURE ONLY: the oracle is the independent CPU reference that
the test suite, the smoke check and the benchmark's CPU-baseline leg compare
the CUDA path against.  Building it is not using it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "alspec_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile oracle/alspec_oracle.c into oracle/liboracle.so; return its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-Wall", "-Wextra", "-shared", "-fPIC",
           "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
