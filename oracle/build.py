"""Compile the CPU oracle (cplse_oracle.c) into liboracle.so beside it.

Test infrastructure: the product library never links or loads this.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cplse_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_oracle(src: str, lib: str) -> str:
    """gcc, float64 loops kept as written: no fast-math, no FMA contraction."""
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_oracle(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
