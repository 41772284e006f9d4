"""Compile the fp64 CPU oracle (test infrastructure) into oracle/liboracle.so.

Only the tests, the smoke check and the bench's CPU-baseline leg load the
result. Building it is part of the repository's build step; using it is not
part of the product path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "parallax_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_source(src: str, out: str) -> str:
    """gcc -O2 -fopenmp -shared: one C file to one shared library."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-Wall", "-Wextra", "-o", out + ".tmp", src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    return compile_source(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
