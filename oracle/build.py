"""Compile the fp64 CPU oracle (plain C, gcc) into oracle/_build/.

Test infrastructure: the product never loads the library this builds.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libkda_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle shared library if it is missing or stale; return its path."""
    os.makedirs(OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    # -O2 without -ffast-math: the oracle keeps IEEE fp64 semantics.
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-fno-fast-math",
           "-ffp-contract=off", "-o", LIB, SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
