"""Compile the C oracle into oracle/_build/libnf4oracle.so.

Test infrastructure: the oracle is the reference the CUDA library is tested
against and is never part of its product path. Building it is not using it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nf4_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libnf4oracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
    "-shared", "-fPIC", "-Wall", "-Wextra", "-Wno-unused-parameter",
]


def build(force: bool = False) -> str:
    """Build the oracle library if missing or older than its source; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
