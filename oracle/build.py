"""Compile the scalar CPU oracle (mxfp4_oracle.c) into liboracle.so with gcc.

The oracle is test infrastructure; building it is part of the build check so
that the tests find it ready. The flags keep IEEE fp32 semantics: no fast-math
and no contraction of a*b+c into an FMA.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mxfp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared",
        "-fno-fast-math", "-ffp-contract=off", "-fno-strict-aliasing",
        "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
