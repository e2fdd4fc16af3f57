"""Compile the fp64 CPU oracle (plain C, gcc, OpenMP) into oracle/liboracle.so.

The oracle is test infrastructure: it is compiled with the package, and only the tests, the smoke
check and the benchmark's CPU-baseline leg use it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_to(src: str, lib: str) -> str:
    """Compile the C source `src` into the shared library `lib` with the oracle's flags."""
    cmd = ["gcc", "-O3", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
           "-Wall", "-Wextra", "-o", lib + ".tmp", src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_to(SRC, LIB)


if __name__ == "__main__":
    print(build(force=True))
