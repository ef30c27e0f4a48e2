"""Build the CPU oracle's shared library (liboracle.so) with gcc.

Test infrastructure: the oracle is built next to its sources and loaded only by the tests,
the package smoke check and the bench's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "llvq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    hdr = os.path.join(HERE, "llvq_oracle.h")
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr))):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off: every product and sum rounds on its own, as written (fma() where written)
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-Wall", "-Wextra", "-fPIC", "-shared",
           "-o", tmp, SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
