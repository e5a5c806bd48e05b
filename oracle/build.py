"""Compile the CPU oracle (``ep_oracle.c``) into ``libep_oracle.so`` next to it.

Test infrastructure: the oracle is built and loaded only by the tests, the
smoke check and the benchmark's CPU-baseline leg.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "libep_oracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared",
    # one IEEE-754 binary32 operation per C operator: no contraction into FMA,
    # no excess precision, no fast-math
    "-ffp-contract=off", "-fexcess-precision=standard", "-fno-fast-math",
    "-Wall", "-Wextra",
]


def build(force: bool = False, verbose: bool = False) -> str:
    """Build the oracle library if missing or older than its source; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)
            and os.path.getmtime(LIB) >= os.path.getmtime(__file__)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
