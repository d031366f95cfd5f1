"""Compile the oracle's C source into oracle/_build/libzero3_ref.so.

Test infrastructure: the oracle is built here so that tests, the smoke check
and the benchmark's CPU-baseline leg can load it.  The flags keep every float
operation a single IEEE-754 binary32 operation: no FMA contraction, no
fast-math reassociation.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zero3_ref.c")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libzero3_ref.so")

CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
          "-Wall", "-Wextra", "-Werror", "-fPIC", "-shared"]


def is_stale() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    """Compile the oracle library if it is missing or older than its source."""
    if force or is_stale():
        os.makedirs(OUT_DIR, exist_ok=True)
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
