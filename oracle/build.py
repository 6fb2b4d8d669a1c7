"""Builds the fp64 CPU oracle (``mla_oracle.c``) into ``liboracle_mla.so``.

Test infrastructure only: the oracle library is loaded by the tests, the smoke
check and the benchmark's CPU-baseline leg, never by the CUDA path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mla_oracle.c")
LIB = os.path.join(HERE, "liboracle_mla.so")


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # -O2 without fast-math: IEEE semantics, no reassociation of the sums.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
