"""Build the CPU oracle library (test infrastructure only).

Compiles ``mla_oracle.cpp`` into ``libmla_oracle.so`` next to it with plain
single-precision SSE arithmetic: no fused multiply-add (``-ffp-contract=off``),
no fast-math, no ``-march`` that could enable FMA.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mla_oracle.cpp")
LIB = os.path.join(HERE, "libmla_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fno-finite-math-only", "-Wall", "-Wextra", "-shared", "-fPIC", "-pthread",
           SRC, "-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
