"""Builds the CPU oracle (plain C, OpenMP) into oracle/libmoe_oracle.so.

Test infrastructure only; the product library never links it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
LIB = os.path.join(HERE, "libmoe_oracle.so")

CFLAGS = ["-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
          "-fPIC", "-shared", "-Wall", "-Wno-unknown-pragmas"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB)
    return LIB


def build_mutant(mutant: int, out_dir: str) -> str:
    """A copy of the oracle with one known mistake planted (ORACLE_MUTANT);
    for the test that shows the pins catch it.  Never used elsewhere."""
    lib = os.path.join(out_dir, "libmoe_oracle_mutant%d.so" % mutant)
    subprocess.check_call(["gcc", *CFLAGS, "-DORACLE_MUTANT=%d" % mutant, "-o", lib, SRC, "-lm"])
    return lib


if __name__ == "__main__":
    print(build(force=True))
