"""Builds the CPU oracle (oracle.c) into liboracle.so next to this file.

Test infrastructure: plain gcc, -O2, no fast-math and no FMA contraction, so
every fp64 operation in the oracle rounds exactly as written.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_to(src: str, lib: str) -> str:
    """Compile one copy of the oracle source into a shared library."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", lib, src, "-lm"]
    subprocess.run(cmd, check=True)
    return lib


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force=True))
