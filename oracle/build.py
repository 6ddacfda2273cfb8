"""Compile the CPU oracle (plain C, OpenMP) into ``oracle/liboracle.so``.

Test infrastructure: the oracle is only ever loaded by the tests, the smoke check and the
benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


# IEEE semantics: no contraction of a*b+c into fma, no fast-math
CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def compile_to(src: str, out: str) -> str:
    """Compile one oracle source file into the shared library `out`."""
    subprocess.run(["gcc", *CFLAGS, "-o", out, src, "-lm"], check=True)
    return out


def build(force: bool = False) -> str:
    """Build liboracle.so if it is missing or older than its source; return its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    compile_to(SRC, LIB + ".tmp")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
