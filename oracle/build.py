"""Compile the C oracle into oracle/libmxfp4_oracle.so.

Test infrastructure: the oracle is only ever loaded by tests/, the smoke check
and the CPU-baseline leg of bench.py.  Building it is not using it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mxfp4_oracle.c")
LIB = os.path.join(HERE, "libmxfp4_oracle.so")

# -ffp-contract=off: no FMA contraction, every float operation rounds as written.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-fopenmp"]


def build(force: bool = False, mutant: int = 0, out: str | None = None) -> str:
    """Build the oracle (or, for the mutation tests, the oracle with planted
    mistake number `mutant` into `out`) and return the library path."""
    lib = out or LIB
    if not force and not mutant and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    cmd = ["gcc", *CFLAGS, *([f"-DORC_MUTANT={mutant}"] if mutant else []), SRC, "-o", lib + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
