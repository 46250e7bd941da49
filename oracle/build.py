"""Compile the fp64 CPU oracle (test infrastructure) into oracle/_hs2_oracle.so.

Plain gcc, -O2 without fast-math so every floating-point operation is the
IEEE double operation the source states; OpenMP only splits independent work.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hs2_oracle.c")
OUT = os.path.join(HERE, "_hs2_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           "-std=c11", "-Wall", "-o", OUT + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
