"""Compile the oracle's C source into oracle/libdg_oracle.so (gcc, OpenMP, no fast-math).

The oracle is test infrastructure: building it is part of ``build()`` so the checker exists on
every machine, but only the tests, the smoke check and the CPU-baseline leg of the benchmark load it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dg_oracle.c")
LIB = os.path.join(HERE, "libdg_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wno-unknown-pragmas",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
