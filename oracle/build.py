"""Compile the CPU oracle (plain C, fp64) into oracle/liboracle_rat.so.

Test infrastructure: the tests, the smoke check and the benchmark's CPU-baseline
leg load the result; the product library never does.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "rat_oracle.c")
LIB = os.path.join(HERE, "liboracle_rat.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    # -ffp-contract=off: no fused multiply-add contraction, each step rounds in
    # IEEE double exactly as written.
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
