"""Compile the fp64 oracle (plain C) into oracle/liboracle.so.

Test infrastructure: building the checker is not using it.  No
-ffast-math: the oracle must keep IEEE fp64 semantics.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "drr_oracle.c")
LIB = os.environ.get("DRR_ORACLE_LIB") or os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-o", LIB, SRC, "-lm", "-lpthread"]
    subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
