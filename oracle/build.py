"""Builds the CPU oracle (test infrastructure) into oracle/libkvq_oracle.so with gcc.

Flags: -O2 -ffp-contract=off -fno-fast-math so that every fp32 expression rounds once per
operation, exactly as written in kvq_oracle.c.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
LIB = os.path.join(HERE, "libkvq_oracle.so")


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "kvq_oracle.h")]
    if not force and os.path.exists(LIB) and all(
        os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps
    ):
        return LIB
    cmd = [
        "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
        "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm",
    ]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
