"""Compile the CPU oracle (test infrastructure) into oracle/liboracle.so.

The flags keep binary32 arithmetic IEEE single precision with no FMA
contraction, so the oracle's MSD expansion is evaluated exactly in the order
the method's equations print it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "w4a16_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
         "-fPIC", "-shared", "-std=c11", "-Wall"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *FLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
