"""Compile the CPU oracle (test infrastructure) into oracle/libmoonep_oracle.so.

The oracle is plain C11 built with gcc.  ``-ffp-contract=off`` keeps every
binary32 multiply and add separately rounded; the single fused step of the
combine calls ``fmaf`` explicitly.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moonep_oracle.c")
LIB = os.path.join(HERE, "libmoonep_oracle.so")


def needs_build() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-Wall", "-Wextra", "-shared", "-fPIC", SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
