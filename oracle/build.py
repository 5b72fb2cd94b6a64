"""Compile the float64 oracle (plain C + OpenMP) into oracle/liboracle.so.

Test infrastructure only: nothing in the CUDA library builds, links or loads this.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gla_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build_mutant(n: int, out_dir: str) -> str:
    """A copy of the oracle with planted mistake number n (tests only)."""
    out = os.path.join(out_dir, f"liboracle_mutant{n}.so")
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", f"-DORACLE_MUTANT={n}",
           "-o", out, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
