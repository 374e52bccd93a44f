"""Build the fp64 CPU oracle (oracle/liboracle.so) with gcc.

Test infrastructure: the oracle is compiled so that the tests, the smoke check
and the CPU-baseline leg of the benchmark can call it; the product library
never links it.  Flags keep IEEE semantics: no fast-math and no contraction
of a*b+c into fused multiply-adds, so every step rounds as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "muon_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-fno-finite-math-only",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
