"""Build the CPU oracle (oracle.c -> liboracle.so) with gcc.

Test infrastructure: the library built here is loaded only by tests/,
__graft_entry__.smoke() and the CPU legs of bench.py. Flags keep the
arithmetic IEEE: no fast-math and no contraction of a*b+c into fused
multiply-adds (the oracle's fused steps are explicit fmaf calls).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-frounding-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
