"""Builds the CPU oracle shared library (test infrastructure only).

``build()`` compiles ``mmf_oracle.c`` with gcc into ``libmmf_oracle.so`` next
to this file.  ``build(src=..., out=...)`` compiles another copy of the source,
which the test suite uses to plant a mistake in a scratch copy of the oracle
and check that its pins catch it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mmf_oracle.c")
LIB = os.path.join(HERE, "libmmf_oracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared",
    # fp32 steps must round exactly as written: no FMA contraction, no fast-math
    "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
    "-fopenmp",
]


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    hdr = os.path.join(HERE, "mmf_oracle.h")
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return out
    cmd = ["gcc", *CFLAGS, "-I", HERE, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
